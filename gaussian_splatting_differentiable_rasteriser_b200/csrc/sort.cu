// Tile lists: order the (Gaussian, tile) entries by tile, then depth, then
// index, and extract per-tile ranges.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), section "Why tiling, and the five stages": count -> scan
// -> scatter -> sort by depth within each tile, equal keys broken by the
// smaller id; each tile's range closes where the next tile begins.
//
// Design (B200): the order (tile, depth, index) is produced by two stable
// radix sorts of 32-bit keys instead of one sort of 64-bit (tile | depth)
// keys over all entries:
//   1. compact the visible Gaussians in index order as
//      (float_bits(depth) - depth_min, index); positive float32 bit patterns
//      order like the floats, so this key orders by depth exactly;
//   2. sort them by that key (ceil(depth_bits / 8) passes, typically 3, over
//      the visible Gaussians only - about 2.2x fewer items than entries);
//   3. duplicate in that depth order: one (tile, index) entry per touched
//      tile; a count kernel sums the tiles of each chunk of Gaussians and a
//      scan turns the sums into each chunk's output offset;
//   4. sort the entries by tile (ceil(tile_bits / 8) passes, 2 at 1080p).
// Every step is stable, so equal depth keys stay in index order and each
// tile's entries stay in (depth, index) order: the same order as one sort by
// (tile, depth) of entries emitted in index order, with about half the bytes
// moved (16 B per item and pass instead of 24, 5 passes over fewer items).
//
// Each radix pass is reduce-then-scan, three launches with no wait between
// CTAs: an upsweep counts each 4096-key chunk's digits (and adds them to the
// pass's digit totals), a scan turns the per-chunk counts of each digit into
// global offsets, and a downsweep ranks its chunk's keys stably in shared
// memory (per-warp digit counters, ballot ranking) and scatters them through
// shared memory, so the global writes are runs of consecutive addresses. The
// upsweep re-reads the keys (4 B of the pass's 20 B per item); at the sizes of
// a training step they mostly come from L2. A single-pass decoupled look-back
// avoids that read but serialises the CTAs of a wave: the prefix frontier
// advances a few CTAs per L2 round trip, which bounded that design at these
// sizes.
#include <algorithm>

#include "gs_kernels.cuh"

namespace gs {

namespace {

// ---------------------------------------------------------------- compact --
// Each CTA compacts kCompactBlocks consecutive preprocess blocks (one Gaussian
// of each per thread), with all their loads in flight together.
constexpr int kCompactBlocks = 4;

__global__ void __launch_bounds__(kGaussBlock) compact_kernel(CompactArgs a) {
  chain_wait();
  chain_release();
  __shared__ uint32_t s_warp[kCompactBlocks][kGaussBlock / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kCompactBlocks;
  bool vis[kCompactBlocks];
  uint32_t key[kCompactBlocks], pre[kCompactBlocks], m[kCompactBlocks];
#pragma unroll
  for (int u = 0; u < kCompactBlocks; ++u) {
    const int64_t i = (b0 + u) * kGaussBlock + threadIdx.x;
    vis[u] = i < a.n && a.touched[i] != 0u;
    key[u] = i < a.n ? __float_as_uint(a.depth[i]) - a.depth_min : 0u;
    pre[u] = (b0 + u) * kGaussBlock < a.n ? a.visible_prefix[b0 + u] : 0u;
  }
#pragma unroll
  for (int u = 0; u < kCompactBlocks; ++u) {
    m[u] = __ballot_sync(0xffffffffu, vis[u]);
    if (lane == 0) s_warp[u][warp] = __popc(m[u]);
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kCompactBlocks; ++u) {
    if (!vis[u]) continue;
    uint32_t before = 0;
    for (int k = 0; k < warp; ++k) before += s_warp[u][k];
    const int64_t off = static_cast<int64_t>(pre[u]) + before + __popc(m[u] & ((1u << lane) - 1u));
    if (off >= a.max_out) {
      record_error(a.err, kErrIndexRange);
      continue;
    }
    a.keys[off] = key[u];
    a.vals[off] = static_cast<uint32_t>((b0 + u) * kGaussBlock + threadIdx.x);
  }
}

// -------------------------------------------------------------- duplicate --
// floor(n / d) for n < 2^22 and 0 < d: n and d are exact in float32, the
// fast quotient is within 2 ulp, i.e. within 1 of n / d below 2^22, so the
// truncated quotient is off by at most one, which one correction step fixes.
__device__ __forceinline__ uint32_t div_small(uint32_t n, uint32_t d) {
  uint32_t q = static_cast<uint32_t>(__fdividef(static_cast<float>(n), static_cast<float>(d)));
  const int32_t r = static_cast<int32_t>(n - q * d);
  if (r < 0) --q;
  else if (static_cast<uint32_t>(r) >= d) ++q;
  return q;
}

// Tiles touched by each chunk of kDupItems Gaussians in depth order (the
// duplicate's CTA granularity): one CTA per chunk, one sum per chunk.
__global__ void __launch_bounds__(kDupThreads) dup_count_kernel(const uint32_t* order, const uint32_t* touched,
                                                                int64_t count, uint32_t* chunk_tiles) {
  chain_wait();
  chain_release();
  __shared__ uint32_t s_warp[kDupThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kDupItems;
  uint32_t sum = 0;
#pragma unroll 4
  for (int j = 0; j < kDupPerThread; ++j) {
    const int64_t idx = base + static_cast<int64_t>(j) * kDupThreads + tid;
    if (idx < count) sum += __ldg(touched + __ldg(order + idx));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_warp[warp] = sum;
  __syncthreads();
  if (tid == 0) {
    uint32_t t = 0;
#pragma unroll
    for (int k = 0; k < kDupThreads / 32; ++k) t += s_warp[k];
    chunk_tiles[blockIdx.x] = t;
  }
}

// Items are warp-striped: item j of lane l of warp w is the CTA's item
// 32 (kDupPerThread w + j) + l, so the order reads are coalesced and, for a
// given j, the lanes' output runs are adjacent in memory.
__global__ void __launch_bounds__(kDupThreads) duplicate_kernel(DuplicateArgs a) {
  chain_wait();
  chain_release();
  __shared__ uint32_t s_warp[kDupThreads / 32];
  __shared__ uint32_t s_pre[kDupThreads / 32][kDupPerThread][32];  // items' offsets in the warp's run
  __shared__ uint32_t s_gid[kDupThreads / 32][kDupPerThread][32];  // items' Gaussians
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tile = blockIdx.x;
  const int64_t wbase = tile * kDupItems + static_cast<int64_t>(warp) * (32 * kDupPerThread);
  uint32_t gid[kDupPerThread];
  uint2 rc[kDupPerThread];
#pragma unroll
  for (int j = 0; j < kDupPerThread; ++j) {
    const int64_t idx = wbase + 32 * j + lane;
    gid[j] = idx < a.count ? __ldg(a.order + idx) : 0u;
    s_gid[warp][j][lane] = gid[j];
  }
#pragma unroll
  for (int j = 0; j < kDupPerThread; ++j) {
    const int64_t idx = wbase + 32 * j + lane;
    // x0 | x1 << 16, y0 | y1 << 16; an empty rect (x1 < x0) for padding items
    rc[j] = idx < a.count ? __ldg(a.rect + gid[j]) : make_uint2(1u, 1u);
  }
  // exclusive prefix of the tiles touched in (j, lane) order inside the warp
  uint32_t run = 0;
#pragma unroll
  for (int j = 0; j < kDupPerThread; ++j) {
    const uint32_t w = (rc[j].x >> 16) + 1u - (rc[j].x & 0xffffu);
    const uint32_t h = (rc[j].y >> 16) + 1u - (rc[j].y & 0xffffu);
    const uint32_t c = w * h;
    uint32_t v = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    s_pre[warp][j][lane] = run + v - c;
    run += __shfl_sync(0xffffffffu, v, 31);
  }
  if (lane == 0) s_warp[warp] = run;
  __syncthreads();
  uint32_t before = 0;
#pragma unroll
  for (int k = 0; k < kDupThreads / 32; ++k) before += k < warp ? s_warp[k] : 0u;
  // this chunk's first entry: the exclusive prefix of the chunks' tile counts
  const uint64_t off0 = static_cast<uint64_t>(__ldg(a.chunk_offsets + tile)) + before;
  if (off0 + run > static_cast<uint64_t>(a.max_entries)) {
    if (lane == 0 && run) record_error(a.err, kErrIndexRange);
    return;
  }
  // The warp writes each group j of 32 items' entries together. When every
  // item of the group touches at most 2 tiles, each lane writes its own
  // entries (adjacent to its neighbours'). Otherwise output o of the group
  // goes to lane o mod 32, which finds the item that owns it by a binary
  // search over the lanes' exclusive offsets: every store of the warp is then
  // one run of 32 consecutive entries, however unevenly the tiles are spread
  // over the items (a few large Gaussians touch hundreds of tiles).
  // The items come back from shared memory (offsets, Gaussians) and the
  // cache (rects, fetched one group ahead) rather than staying in registers,
  // so this loop is not unrolled and the kernel keeps its occupancy.
  const uint32_t tiles_x = static_cast<uint32_t>(a.tiles_x);
  auto rect_of = [&](int j) {
    return wbase + 32 * j + lane < a.count ? __ldg(a.rect + s_gid[warp][j][lane]) : make_uint2(1u, 1u);
  };
  uint2 r_next = rect_of(0);
#pragma unroll 1
  for (int j = 0; j < kDupPerThread; ++j) {
    const uint32_t g = s_gid[warp][j][lane];
    const uint2 r = r_next;
    if (j + 1 < kDupPerThread) r_next = rect_of(j + 1);
    const uint32_t p = s_pre[warp][j][lane];
    const uint32_t gstart = __shfl_sync(0xffffffffu, p, 0);
    const uint32_t excl = p - gstart;  // this lane's first output in the group
    const uint32_t x0 = r.x & 0xffffu, y0 = r.y & 0xffffu;
    const uint32_t w = (r.x >> 16) + 1u - x0;
    const uint32_t h = (r.y >> 16) + 1u - y0;  // padding items: w = h = 0
    const uint32_t last_excl = __shfl_sync(0xffffffffu, excl, 31);
    const uint32_t last_c = __shfl_sync(0xffffffffu, w * h, 31);
    const uint32_t group_total = last_excl + last_c;
    uint32_t* keys = a.keys + off0 + gstart;
    uint32_t* vals = a.vals + off0 + gstart;
    if (__all_sync(0xffffffffu, w * h <= 2u)) {
      // every item touches at most 2 tiles: each lane writes its own (adjacent) entries
      for (uint32_t k = 0; k < w * h; ++k) {
        keys[excl + k] = w == 1u ? (y0 + k) * tiles_x + x0 : y0 * tiles_x + x0 + k;
        vals[excl + k] = g;
      }
      continue;
    }
    for (uint32_t ob = 0; ob < group_total; ob += 32) {
      const uint32_t o = ob + static_cast<uint32_t>(lane);
      // owner = the highest lane whose first output is <= o (it has a non-empty rect)
      int owner = 0;
#pragma unroll
      for (int step = 16; step > 0; step >>= 1) {
        const uint32_t e = __shfl_sync(0xffffffffu, excl, owner + step);
        if (e <= o) owner += step;
      }
      const uint32_t oe = __shfl_sync(0xffffffffu, excl, owner);
      const uint32_t ow = __shfl_sync(0xffffffffu, w, owner);
      const uint32_t ox0 = __shfl_sync(0xffffffffu, x0, owner);
      const uint32_t oy0 = __shfl_sync(0xffffffffu, y0, owner);
      const uint32_t og = __shfl_sync(0xffffffffu, g, owner);
      if (o < group_total) {
        const uint32_t local = o - oe;
        const uint32_t dy = group_total < (1u << 22) ? div_small(local, ow) : local / ow;
        keys[o] = (oy0 + dy) * tiles_x + ox0 + (local - dy * ow);
        vals[o] = og;
      }
    }
  }
}

// ---------------------------------------------------------------- upsweep --
// Digit counts of one pass for the chunk of kSortTileKeys keys of this CTA,
// digit-major (counts[d * chunks + chunk]), and the pass's digit totals
// (hist[d], added with one atomic per digit and CTA).
__global__ void __launch_bounds__(kSortThreads) upsweep_kernel(const uint32_t* keys, int64_t n, int shift,
                                                               int64_t chunks, uint32_t* counts,
                                                               uint32_t* hist) {
  chain_wait();
  chain_release();
  __shared__ uint32_t s_h[kSortThreads / 32][kRadix];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSortTileKeys;
  const bool full = base + kSortTileKeys <= n;
  // A full chunk's keys are loaded (16 bytes at a time: the chunk starts at a
  // multiple of kSortTileKeys keys) before the counters are cleared, so the
  // loads are in flight meanwhile.
  uint4 q[kSortItems / 4];
  if (full) {
#pragma unroll
    for (int k = 0; k < kSortItems / 4; ++k)
      q[k] = __ldg(reinterpret_cast<const uint4*>(keys + base + 4 * (static_cast<int64_t>(k) * kSortThreads + tid)));
  }
  for (int k = tid; k < (kSortThreads / 32) * kRadix; k += kSortThreads) (&s_h[0][0])[k] = 0;
  __syncthreads();
  if (full) {
#pragma unroll
    for (int k = 0; k < kSortItems / 4; ++k) {
      atomicAdd(&s_h[warp][(q[k].x >> shift) & 0xffu], 1u);
      atomicAdd(&s_h[warp][(q[k].y >> shift) & 0xffu], 1u);
      atomicAdd(&s_h[warp][(q[k].z >> shift) & 0xffu], 1u);
      atomicAdd(&s_h[warp][(q[k].w >> shift) & 0xffu], 1u);
    }
  } else {
#pragma unroll
    for (int k = 0; k < kSortItems / 4; ++k) {
      const int64_t idx = base + 4 * (static_cast<int64_t>(k) * kSortThreads + tid);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (idx + j < n) atomicAdd(&s_h[warp][(__ldg(keys + idx + j) >> shift) & 0xffu], 1u);
    }
  }
  __syncthreads();
  for (int d = tid; d < kRadix; d += kSortThreads) {
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kSortThreads / 32; ++w) c += s_h[w][d];
    counts[static_cast<int64_t>(d) * chunks + blockIdx.x] = c;
    if (c) atomicAdd(&hist[d], c);
  }
}

// ------------------------------------------------------------------- scan --
// CTA d: the global offsets of digit d in every chunk, in place over its
// counts: the keys of all smaller digits (the totals hist[0..d)) come first,
// then digit d's keys of the chunks before.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) scan_digits_kernel(uint32_t* counts, int64_t chunks,
                                                                    const uint32_t* hist) {
  chain_wait();
  chain_release();
  __shared__ uint32_t s_warp[kScanThreads / 32];
  __shared__ uint32_t s_carry;
  const int d = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (warp == 0) {
    uint32_t b = 0;
#pragma unroll
    for (int u = 0; u < kRadix / 32; ++u) {  // d < kRadix: all loads in flight at once
      const int k = lane + 32 * u;
      b += k < d ? hist[k] : 0u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xffffffffu, b, o);
    if (lane == 0) s_carry = b;
  }
  __syncthreads();
  uint32_t* row = counts + static_cast<int64_t>(d) * chunks;
  for (int64_t start = 0; start < chunks; start += 4 * kScanThreads) {
    const int64_t i0 = start + 4 * static_cast<int64_t>(tid);
    uint32_t v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = i0 + j < chunks ? row[i0 + j] : 0u;
    const uint32_t t = v[0] + v[1] + v[2] + v[3];
    uint32_t inc = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    uint32_t before = s_carry, total = 0;
#pragma unroll 4
    for (int w = 0; w < kScanThreads / 32; ++w) {
      const uint32_t x = s_warp[w];
      before += w < warp ? x : 0u;
      total += x;
    }
    uint32_t run = before + inc - t;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (i0 + j < chunks) row[i0 + j] = run;
      run += v[j];
    }
    __syncthreads();
    if (tid == 0) s_carry += total;
    __syncthreads();
  }
}

// -------------------------------------------------------------- downsweep --
struct DownsweepArgs {
  const uint32_t* keys_in;
  const uint32_t* vals_in;
  uint32_t* keys_out;
  uint32_t* vals_out;
  int64_t n;
  int shift;
  int digit_bits;          // significant bits of this pass's digit (1..8)
  const uint32_t* offsets; // [256][chunks]: global first slot of each digit for each chunk
  int64_t chunks;
  uint32_t* err;
};

// Shared memory of one downsweep CTA (dynamic: above the 48 KB static limit).
struct DownsweepSmem {
  uint32_t keys[kSortTileKeys];
  uint32_t vals[kSortTileKeys];
  uint32_t whist[kSortThreads / 32][kRadix];  // per-warp digit counts, then CTA slots
  uint32_t out[kRadix];                       // global slot minus CTA slot of each digit
  uint32_t wsum[kRadix / 32];
};

// kBits: significant bits of this pass's digit; kFull: the chunk holds
// kSortTileKeys keys (every chunk but the last), so no key needs a bounds test.
template <int kBits, bool kFull>
__device__ __forceinline__ void downsweep_chunk(const DownsweepArgs& a, DownsweepSmem& sm, int64_t chunk) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t base = chunk * kSortTileKeys;
  const int valid_n = kFull ? kSortTileKeys : static_cast<int>(a.n - base);
  const uint32_t lt_mask = (1u << lane) - 1u;
  auto& whist = sm.whist;
  for (int k = tid; k < (kSortThreads / 32) * kRadix; k += kSortThreads) (&whist[0][0])[k] = 0;
  // The chunk's global slot of each digit, read early: its latency overlaps the ranking.
  const bool owns_digit = tid < kRadix;
  const uint32_t gbase = owns_digit && tid < (1 << kBits) ? __ldg(a.offsets + tid * a.chunks + chunk) : 0u;

  // Load: warp w owns the kSortItems * 32 consecutive keys from base + w kSortItems 32;
  // item j of lane l is key 32 j + l of that run (coalesced, and in key order j-major).
  const int wbase = warp * (kSortItems * 32);
  uint32_t key[kSortItems], val[kSortItems], dig[kSortItems];
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int e = wbase + 32 * j + lane;
    if (kFull || e < valid_n) {
      key[j] = __ldg(a.keys_in + base + e);
      val[j] = __ldg(a.vals_in + base + e);
    } else {
      key[j] = 0u;
      val[j] = 0u;
    }
    dig[j] = (key[j] >> a.shift) & ((1u << kBits) - 1u);
  }
  __syncthreads();  // counters zeroed

  // Stable rank inside the warp: items in key order, lanes in lane order. The
  // lanes holding the same digit come from one ballot per digit bit.
  uint32_t rank[kSortItems];
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const bool valid = kFull || wbase + 32 * j + lane < valid_n;
    uint32_t peers = kFull ? 0xffffffffu : __ballot_sync(0xffffffffu, valid);
#pragma unroll
    for (int bit = 0; bit < kBits; ++bit) {
      const uint32_t on = 0u - ((dig[j] >> bit) & 1u);
      const uint32_t vote = __ballot_sync(0xffffffffu, on != 0u);
      peers &= ~(vote ^ on);
    }
    const uint32_t b = valid ? whist[warp][dig[j]] : 0u;
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) whist[warp][dig[j]] = b + __popc(peers);
    __syncwarp();
    rank[j] = b + __popc(peers & lt_mask);
  }
  __syncthreads();

  // Per digit (thread d): the CTA-wide exclusive scan of the digit counts, then
  // each warp's first CTA slot of the digit, and global slot minus CTA slot.
  uint32_t count = 0, v = 0;
  if (owns_digit) {
#pragma unroll
    for (int w = 0; w < kSortThreads / 32; ++w) count += whist[w][tid];
    v = count;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) sm.wsum[warp] = v;
  }
  __syncthreads();
  if (owns_digit) {
    uint32_t start = v - count;
    for (int k = 0; k < warp; ++k) start += sm.wsum[k];
    sm.out[tid] = gbase - start;
#pragma unroll
    for (int w = 0; w < kSortThreads / 32; ++w) {
      const uint32_t c = whist[w][tid];
      whist[w][tid] = start;
      start += c;
    }
  }
  __syncthreads();

  // Scatter into shared memory in digit order, then out in runs of consecutive slots.
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    if (kFull || wbase + 32 * j + lane < valid_n) {
      const uint32_t pos = whist[warp][dig[j]] + rank[j];
      if (pos >= static_cast<uint32_t>(kSortTileKeys)) {
        record_error(a.err, kErrIndexRange);
        continue;
      }
      sm.keys[pos] = key[j];
      sm.vals[pos] = val[j];
    }
  }
  __syncthreads();
  for (int k = tid; k < valid_n; k += kSortThreads) {
    const uint32_t kk = sm.keys[k];
    const uint32_t dst = sm.out[(kk >> a.shift) & ((1u << kBits) - 1u)] + static_cast<uint32_t>(k);
    if (static_cast<int64_t>(dst) >= a.n) {
      record_error(a.err, kErrIndexRange);
      continue;
    }
    a.keys_out[dst] = kk;
    a.vals_out[dst] = sm.vals[k];
  }
}

template <int kBits>
__global__ void __launch_bounds__(kSortThreads, GS_SORT_MINB) downsweep_kernel(DownsweepArgs a) {
  chain_wait();
  chain_release();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  DownsweepSmem& sm = *reinterpret_cast<DownsweepSmem*>(smem_raw);
  const int64_t chunk = blockIdx.x;
  if ((chunk + 1) * kSortTileKeys <= a.n)
    downsweep_chunk<kBits, true>(a, sm, chunk);
  else
    downsweep_chunk<kBits, false>(a, sm, chunk);
}

template <int kBits>
cudaError_t launch_downsweep(const DownsweepArgs& o, unsigned chunks, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(downsweep_kernel<kBits>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sizeof(DownsweepSmem)));
  if (e != cudaSuccess) return e;
  return launch_chained(downsweep_kernel<kBits>, dim3(chunks), dim3(kSortThreads), sizeof(DownsweepSmem), st, o);
}

cudaError_t launch_downsweep_bits(const DownsweepArgs& o, int bits, unsigned chunks, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_downsweep<1>(o, chunks, st);
    case 2: return launch_downsweep<2>(o, chunks, st);
    case 3: return launch_downsweep<3>(o, chunks, st);
    case 4: return launch_downsweep<4>(o, chunks, st);
    case 5: return launch_downsweep<5>(o, chunks, st);
    case 6: return launch_downsweep<6>(o, chunks, st);
    case 7: return launch_downsweep<7>(o, chunks, st);
    default: return launch_downsweep<8>(o, chunks, st);
  }
}

// ------------------------------------------------------------------ ranges --
// Each thread looks at kRangeItems consecutive sorted entries (two 16-byte
// loads) and the one before them; every change of tile between neighbours
// closes the previous tile's range and opens the next one's.
constexpr int kRangeItems = 8;

__global__ void __launch_bounds__(256) ranges_kernel(const uint32_t* keys, int64_t n, uint2* ranges,
                                                     int64_t num_tiles) {
  chain_wait();
  chain_release();
  const int64_t i0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * kRangeItems;
  if (i0 >= n) return;
  uint32_t k[kRangeItems];
  if (i0 + kRangeItems <= n) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(keys + i0));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(keys + i0) + 1);
    k[0] = a.x, k[1] = a.y, k[2] = a.z, k[3] = a.w, k[4] = b.x, k[5] = b.y, k[6] = b.z, k[7] = b.w;
  } else {
#pragma unroll
    for (int j = 0; j < kRangeItems; ++j) k[j] = i0 + j < n ? __ldg(keys + i0 + j) : ~0u;
  }
  const uint64_t tiles = static_cast<uint64_t>(num_tiles);
  uint32_t prev = i0 > 0 ? __ldg(keys + i0 - 1) : ~0u;
#pragma unroll
  for (int j = 0; j < kRangeItems; ++j) {
    const int64_t i = i0 + j;
    if (i >= n) break;
    const uint32_t cur = k[j];
    if (cur != prev) {
      if (cur < tiles) ranges[cur].x = static_cast<uint32_t>(i);
      if (prev < tiles) ranges[prev].y = static_cast<uint32_t>(i);
    }
    prev = cur;
  }
  if (i0 + kRangeItems >= n && prev < tiles) ranges[prev].y = static_cast<uint32_t>(n);
}

// The tiles by descending list length, in buckets of equal bit length (the
// order inside a bucket is the atomics' order; a tile's result does not
// depend on when it runs). Taking the longest tiles first keeps a kernel over
// the tiles from ending on a long tile that started late.
constexpr int kOrderThreads = 1024;
__global__ void __launch_bounds__(kOrderThreads) tile_order_kernel(const uint2* ranges, int64_t num_tiles,
                                                                   uint32_t* order) {
  chain_wait();
  chain_release();
  __shared__ uint32_t cnt[33];  // by __clz(length): 0 for the longest, 32 for empty tiles
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  constexpr int kPer = 8;  // tiles per thread and round, loaded together
  constexpr int kRound = kPer * kOrderThreads;
  if (tid < 33) cnt[tid] = 0u;
  // bucket of tile t (33 past the end)
  auto bucket_of = [&](int64_t t) -> uint32_t {
    if (t >= num_tiles) return 33u;
    const uint2 r = ranges[t];
    return __clz(r.y - r.x);
  };
  __syncthreads();
  // Warp w's tiles of a round are [r + 32 (kPer w + j), + 32), j < kPer: the
  // lanes of a warp with the same bucket add to it once.
  for (int64_t r0 = 0; r0 < num_tiles; r0 += kRound) {
    uint32_t b[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) b[j] = bucket_of(r0 + 32 * (kPer * warp + j) + lane);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const unsigned same = __match_any_sync(0xffffffffu, b[j]);
      if (b[j] < 33u && (same & lt) == 0u) atomicAdd(&cnt[b[j]], __popc(same));
    }
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t run = 0u;
    for (int k = 0; k < 33; ++k) {
      const uint32_t c = cnt[k];
      cnt[k] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int64_t r0 = 0; r0 < num_tiles; r0 += kRound) {
    uint32_t b[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) b[j] = bucket_of(r0 + 32 * (kPer * warp + j) + lane);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int64_t t = r0 + 32 * (kPer * warp + j) + lane;
      const unsigned same = __match_any_sync(0xffffffffu, b[j]);
      const int leader = __ffs(same) - 1;
      uint32_t base = 0u;
      if (b[j] < 33u && lane == leader) base = atomicAdd(&cnt[b[j]], __popc(same));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (b[j] < 33u) order[base + __popc(same & lt)] = static_cast<uint32_t>(t);
    }
  }
}

}  // namespace

cudaError_t launch_tile_order(const uint2* ranges, int64_t num_tiles, uint32_t* order, cudaStream_t st) {
  if (num_tiles <= 0) return cudaSuccess;
  return launch_chained(tile_order_kernel, dim3(1), dim3(kOrderThreads), 0, st, ranges, num_tiles, order);
}

cudaError_t launch_compact(const CompactArgs& a, int64_t num_blocks, cudaStream_t st) {
  if (num_blocks == 0) return cudaSuccess;
  return launch_chained(compact_kernel, dim3(static_cast<unsigned>((num_blocks + kCompactBlocks - 1) / kCompactBlocks)),
                        dim3(kGaussBlock), 0, st, a);
}

cudaError_t launch_duplicate(const DuplicateArgs& a, cudaStream_t st) {
  if (a.count == 0) return cudaSuccess;
  const int64_t chunks = (a.count + kDupItems - 1) / kDupItems;
  const unsigned grid = static_cast<unsigned>(chunks);
  // per-chunk tile counts, their exclusive prefix in place (one scan row), then the entries
  cudaError_t e = launch_chained(dup_count_kernel, dim3(grid), dim3(kDupThreads), 0, st, a.order, a.touched, a.count,
                                 a.chunk_offsets);
  if (e == cudaSuccess)
    e = launch_chained(scan_digits_kernel, dim3(1), dim3(kScanThreads), 0, st, a.chunk_offsets, chunks, nullptr);
  if (e == cudaSuccess) e = launch_chained(duplicate_kernel, dim3(grid), dim3(kDupThreads), 0, st, a);
  return e;
}

cudaError_t launch_sort(const SortPlan& plan, const SortBuffers& b, int* out_buf, cudaStream_t st) {
  *out_buf = 0;
  if (plan.n <= 1 || plan.passes == 0) return cudaSuccess;
  cudaError_t e;
  if ((e = cudaMemsetAsync(b.hist, 0, sizeof(uint32_t) * kMaxPasses * kRadix, st)) != cudaSuccess) return e;
  const unsigned chunks = static_cast<unsigned>(plan.tiles);
  int cur = 0;
  for (int p = 0; p < plan.passes; ++p) {
    const int digit_bits = std::min(8, plan.key_bits - 8 * p);
    uint32_t* counts = b.chunk_counts + static_cast<int64_t>(p) * plan.tiles * kRadix;  // [256][chunks]
    uint32_t* hist = b.hist + p * kRadix;
    if ((e = launch_chained(upsweep_kernel, dim3(chunks), dim3(kSortThreads), 0, st, b.keys[cur], plan.n, 8 * p,
                            plan.tiles, counts, hist)) != cudaSuccess)
      return e;
    if ((e = launch_chained(scan_digits_kernel, dim3(1u << digit_bits), dim3(kScanThreads), 0, st, counts, plan.tiles,
                            hist)) != cudaSuccess)
      return e;
    DownsweepArgs o;
    o.keys_in = b.keys[cur];
    o.vals_in = b.vals[cur];
    o.keys_out = b.keys[cur ^ 1];
    o.vals_out = b.vals[cur ^ 1];
    o.n = plan.n;
    o.shift = 8 * p;
    o.digit_bits = digit_bits;
    o.offsets = counts;
    o.chunks = plan.tiles;
    o.err = b.err;
    if ((e = launch_downsweep_bits(o, digit_bits, chunks, st)) != cudaSuccess) return e;
    cur ^= 1;
  }
  *out_buf = cur;
  return cudaSuccess;
}

cudaError_t launch_ranges(const uint32_t* keys, int64_t n, uint2* ranges, int64_t num_tiles,
                          cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(ranges, 0, sizeof(uint2) * num_tiles, st);
  if (e != cudaSuccess || n == 0) return e;
  const int64_t per_block = 256 * kRangeItems;
  return launch_chained(ranges_kernel, dim3(static_cast<unsigned>((n + per_block - 1) / per_block)), dim3(256), 0, st,
                        keys, n, ranges, num_tiles);
}

}  // namespace gs
