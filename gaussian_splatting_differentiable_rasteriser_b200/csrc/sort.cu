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
//      tile, each CTA's output offset found by a decoupled look-back;
//   4. sort the entries by tile (ceil(tile_bits / 8) passes, 2 at 1080p).
// Every step is stable, so equal depth keys stay in index order and each
// tile's entries stay in (depth, index) order: the same order as one sort by
// (tile, depth) of entries emitted in index order, with about half the bytes
// moved (16 B per item and pass instead of 24, 5 passes over fewer items).
//
// Each onesweep pass reads and writes every item once: a CTA ranks 4096 keys
// in shared memory (per-warp digit counters, ballot ranking), publishes its
// digit counts, obtains the exclusive prefix of all earlier CTAs by a
// decoupled look-back whose every wait is bounded, and scatters through shared
// memory so the global writes are runs of consecutive addresses.
#include <algorithm>

#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagPrefix = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1u;
constexpr int kLookbackSpinLimit = 1 << 22;

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- compact --
__global__ void __launch_bounds__(256) compact_kernel(CompactArgs a) {
  __shared__ uint32_t s_warp[8];
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool vis = i < a.n && a.touched[i] != 0u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t m = __ballot_sync(0xffffffffu, vis);
  if (lane == 0) s_warp[warp] = __popc(m);
  __syncthreads();
  if (!vis) return;
  uint32_t before = 0;
  for (int k = 0; k < warp; ++k) before += s_warp[k];
  const int64_t off = static_cast<int64_t>(a.visible_prefix[blockIdx.x]) + before +
                      __popc(m & ((1u << lane) - 1u));
  if (off >= a.max_out) {
    record_error(a.err, kErrIndexRange);
    return;
  }
  a.keys[off] = __float_as_uint(a.depth[i]) - a.depth_min;
  a.vals[off] = static_cast<uint32_t>(i);
}

// -------------------------------------------------------------- duplicate --
// Decoupled look-back over earlier CTAs' status words (flag | value) by one
// warp, 32 predecessors per round; returns the sum of the values before
// `tile`. Every wait is bounded; on giving up it records an error and returns
// what it has.
__device__ __forceinline__ uint32_t warp_lookback(const uint32_t* status, int64_t tile, int lane,
                                                  uint32_t* err) {
  uint32_t excl = 0;
  int64_t t = tile - 1;
  int spins = 0;
  while (t >= 0) {
    const uint32_t w = (t - lane >= 0) ? ld_relaxed(&status[t - lane]) : kFlagPrefix;
    const uint32_t flag = w & ~kValueMask;
    const unsigned not_ready = __ballot_sync(0xffffffffu, flag == 0u);
    const unsigned is_prefix = __ballot_sync(0xffffffffu, flag == kFlagPrefix);
    // lanes usable this round: up to (and including) the first prefix, before the first not-ready
    const unsigned upto_prefix = is_prefix ? ((2u << (__ffs(is_prefix) - 1)) - 1u) : 0xffffffffu;
    const unsigned before_wait = not_ready ? ((1u << (__ffs(not_ready) - 1)) - 1u) : 0xffffffffu;
    const unsigned use = upto_prefix & before_wait;
    uint32_t v = ((use >> lane) & 1u) ? (w & kValueMask) : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    excl += v;
    if (is_prefix && (upto_prefix & ~before_wait) == 0u) break;  // reached a prefix
    t -= __popc(use);
    if (not_ready) {
      if (++spins > kLookbackSpinLimit) {
        record_error(err, kErrLookbackTimeout);
        break;
      }
      __nanosleep(32);
    }
  }
  return excl;
}

// Items are warp-striped: item j of lane l of warp w is the CTA's item
// 32 (kDupPerThread w + j) + l, so the order reads are coalesced and, for a
// given j, the lanes' output runs are adjacent in memory.
__global__ void __launch_bounds__(kDupThreads) duplicate_kernel(DuplicateArgs a) {
  __shared__ uint32_t s_warp[kDupThreads / 32];
  __shared__ uint32_t s_pre[kDupThreads / 32][kDupPerThread][32];  // items' offsets in the warp's run
  __shared__ uint32_t s_gid[kDupThreads / 32][kDupPerThread][32];  // items' Gaussians
  __shared__ uint32_t s_tile, s_excl;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_tile = atomicAdd(a.ticket, 1u);
  __syncthreads();
  const int64_t tile = s_tile;
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
  uint32_t before = 0, total = 0;
#pragma unroll
  for (int k = 0; k < kDupThreads / 32; ++k) {
    before += k < warp ? s_warp[k] : 0u;
    total += s_warp[k];
  }
  uint32_t* st = a.status + tile;
  if (warp == 0) {
    if (lane == 0) st_relaxed(st, (tile == 0 ? kFlagPrefix : kFlagAggregate) | total);
    uint32_t excl = 0;
    if (tile > 0) {
      excl = warp_lookback(a.status, tile, lane, a.err);
      if (lane == 0) st_relaxed(st, kFlagPrefix | (excl + total));
    }
    if (lane == 0) s_excl = excl;
  }
  __syncthreads();
  const uint64_t off0 = static_cast<uint64_t>(s_excl) + before;
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
        const uint32_t dy = local / ow;
        keys[o] = (oy0 + dy) * tiles_x + ox0 + (local - dy * ow);
        vals[o] = og;
      }
    }
  }
}

// ------------------------------------------------------------- histogram --
__global__ void __launch_bounds__(256) histogram_kernel(const uint32_t* keys, int64_t n,
                                                        int passes, uint32_t* hist) {
  __shared__ uint32_t s_hist[kMaxPasses][kRadix];
  for (int k = threadIdx.x; k < kMaxPasses * kRadix; k += blockDim.x) (&s_hist[0][0])[k] = 0;
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint32_t key = keys[i];
    for (int p = 0; p < passes; ++p) atomicAdd(&s_hist[p][(key >> (8 * p)) & 0xffu], 1u);
  }
  __syncthreads();
  for (int p = 0; p < passes; ++p) {
    const uint32_t c = s_hist[p][threadIdx.x];
    if (c) atomicAdd(&hist[p * kRadix + threadIdx.x], c);
  }
}

// Exclusive scan of each pass's digit histogram: one CTA of 256 per pass.
__global__ void __launch_bounds__(256) digit_offsets_kernel(const uint32_t* hist, uint32_t* offsets) {
  __shared__ uint32_t s_warp[8];
  const int p = blockIdx.x, d = threadIdx.x, lane = d & 31, warp = d >> 5;
  const uint32_t c = hist[p * kRadix + d];
  uint32_t v = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  uint32_t before = 0;
  for (int k = 0; k < warp; ++k) before += s_warp[k];
  offsets[p * kRadix + d] = before + v - c;
}

// --------------------------------------------------------------- onesweep --
struct OnesweepArgs {
  const uint32_t* keys_in;
  const uint32_t* vals_in;
  uint32_t* keys_out;
  uint32_t* vals_out;
  int64_t n;
  int shift;
  int digit_bits;                 // significant bits of this pass's digit (1..8)
  const uint32_t* digit_offsets;  // [256] for this pass
  uint32_t* status;               // [tiles][256] for this pass, zeroed
  uint32_t* ticket;               // zeroed
  uint32_t* err;
};

// Shared memory of one onesweep CTA (dynamic: above the 48 KB static limit).
struct OnesweepSmem {
  uint32_t keys[kSortTileKeys];
  uint32_t vals[kSortTileKeys];
  uint32_t whist[kSortThreads / 32][kRadix];  // per-warp digit counts, then offsets
  uint32_t start[kRadix];  // first slot of each digit inside this CTA
  uint32_t base[kRadix];   // first global slot of each digit for this CTA
  uint32_t wsum[kSortThreads / 32];
  uint32_t tile;
};

__global__ void __launch_bounds__(kSortThreads) onesweep_kernel(OnesweepArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  OnesweepSmem& sm = *reinterpret_cast<OnesweepSmem*>(smem_raw);
  uint32_t* s_keys = sm.keys;
  uint32_t* s_vals = sm.vals;
  auto& s_whist = sm.whist;
  uint32_t* s_start = sm.start;
  uint32_t* s_base = sm.base;
  uint32_t* s_wsum = sm.wsum;
  uint32_t& s_tile = sm.tile;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_tile = atomicAdd(a.ticket, 1u);
  for (int k = tid; k < (kSortThreads / 32) * kRadix; k += kSortThreads) (&s_whist[0][0])[k] = 0;
  __syncthreads();
  const uint32_t tile = s_tile;
  const int64_t base = static_cast<int64_t>(tile) * kSortTileKeys;
  const uint32_t lt_mask = (1u << lane) - 1u;

  // Load: warp w owns the 512 consecutive entries [base + 512 w, base + 512 (w + 1)),
  // item j of lane l is entry 32 j + l of that run (coalesced).
  uint32_t key[kSortItems];
  uint32_t val[kSortItems];
  uint32_t rank[kSortItems];
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int64_t idx = base + warp * (kSortItems * 32) + j * 32 + lane;
    if (idx < a.n) {
      key[j] = a.keys_in[idx];
      val[j] = a.vals_in[idx];
    } else {
      key[j] = ~0u;
      val[j] = 0u;
    }
  }
  // Stable rank inside the warp: items in entry order, lanes in lane order.
  // Lanes holding the same digit are found with one ballot per digit bit.
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int64_t idx = base + warp * (kSortItems * 32) + j * 32 + lane;
    const bool valid = idx < a.n;
    const uint32_t d = (key[j] >> a.shift) & 0xffu;
    uint32_t peers = __ballot_sync(0xffffffffu, valid);
#pragma unroll
    for (int bit = 0; bit < 8; ++bit) {
      if (bit >= a.digit_bits) break;
      const bool on = (d >> bit) & 1u;
      const uint32_t vote = __ballot_sync(0xffffffffu, on);
      peers &= on ? vote : ~vote;
    }
    const uint32_t b = valid ? s_whist[warp][d] : 0u;
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) s_whist[warp][d] = b + __popc(peers);
    __syncwarp();
    rank[j] = b + __popc(peers & lt_mask);
  }
  __syncthreads();

  // Per digit: exclusive offsets of each warp, and the CTA total.
  const uint32_t d = tid;  // kSortThreads == kRadix
  uint32_t count = 0;
#pragma unroll
  for (int w = 0; w < kSortThreads / 32; ++w) {
    const uint32_t c = s_whist[w][d];
    s_whist[w][d] = count;
    count += c;
  }
  // Publish this CTA's count before anything else, so later CTAs can proceed.
  uint32_t* st = a.status + static_cast<int64_t>(tile) * kRadix;
  st_relaxed(&st[d], (tile == 0 ? kFlagPrefix : kFlagAggregate) | count);

  // CTA-wide exclusive scan of the digit counts.
  uint32_t v = count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_wsum[warp] = v;
  __syncthreads();
  uint32_t before = 0;
  for (int k = 0; k < warp; ++k) before += s_wsum[k];
  s_start[d] = before + v - count;

  // Decoupled look-back over earlier CTAs for this digit, kWindow predecessors
  // per round: their status words are loaded together, so a run of
  // aggregate-only predecessors costs one memory latency per kWindow CTAs.
  // (When a whole wave of CTAs starts at once, none has its inclusive prefix
  // yet and CTA k of the wave must sum back k aggregates.) Every wait is bounded.
  constexpr int kWindow = 8;
  uint32_t excl = 0;
  if (tile > 0) {
    int64_t t = static_cast<int64_t>(tile) - 1;
    int spins = 0;
    while (t >= 0) {
      uint32_t w[kWindow];
#pragma unroll
      for (int k = 0; k < kWindow; ++k)
        w[k] = (t - k >= 0) ? ld_relaxed(&a.status[(t - k) * kRadix + d]) : kFlagPrefix;
      int used = 0;
      bool stop = false, blocked = false;
#pragma unroll
      for (int k = 0; k < kWindow; ++k) {
        if (stop || blocked) continue;
        const uint32_t flag = w[k] & ~kValueMask;
        if (flag == 0u) {
          blocked = true;
          continue;
        }
        excl += w[k] & kValueMask;
        ++used;
        if (flag == kFlagPrefix) stop = true;
      }
      if (stop) break;
      t -= used;
      if (blocked) {
        if (++spins > kLookbackSpinLimit) {
          record_error(a.err, kErrLookbackTimeout);
          break;
        }
        __nanosleep(32);
      }
    }
    st_relaxed(&st[d], kFlagPrefix | (excl + count));
  }
  s_base[d] = a.digit_offsets[d] + excl;
  __syncthreads();

  // Scatter into shared memory in digit order, then out in runs.
#pragma unroll
  for (int j = 0; j < kSortItems; ++j) {
    const int64_t idx = base + warp * (kSortItems * 32) + j * 32 + lane;
    if (idx < a.n) {
      const uint32_t dj = (key[j] >> a.shift) & 0xffu;
      const uint32_t pos = s_start[dj] + s_whist[warp][dj] + rank[j];
      if (pos >= static_cast<uint32_t>(kSortTileKeys)) {
        record_error(a.err, kErrIndexRange);
        continue;
      }
      s_keys[pos] = key[j];
      s_vals[pos] = val[j];
    }
  }
  __syncthreads();
  const int64_t rem = a.n - base;
  const int tile_n = rem < kSortTileKeys ? static_cast<int>(rem) : kSortTileKeys;
  for (int k = tid; k < tile_n; k += kSortThreads) {
    const uint32_t kk = s_keys[k];
    const uint32_t dk = (kk >> a.shift) & 0xffu;
    const int64_t dst = static_cast<int64_t>(s_base[dk]) + (k - static_cast<int64_t>(s_start[dk]));
    if (dst < 0 || dst >= a.n) {
      record_error(a.err, kErrIndexRange);
      continue;
    }
    a.keys_out[dst] = kk;
    a.vals_out[dst] = s_vals[k];
  }
}

// ------------------------------------------------------------------ ranges --
// Each thread looks at kRangeItems consecutive sorted entries (two 16-byte
// loads) and the one before them; every change of tile between neighbours
// closes the previous tile's range and opens the next one's.
constexpr int kRangeItems = 8;

__global__ void __launch_bounds__(256) ranges_kernel(const uint32_t* keys, int64_t n, uint2* ranges,
                                                     int64_t num_tiles) {
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

}  // namespace

cudaError_t launch_compact(const CompactArgs& a, int64_t num_blocks, cudaStream_t st) {
  if (num_blocks == 0) return cudaSuccess;
  compact_kernel<<<static_cast<unsigned>(num_blocks), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_duplicate(const DuplicateArgs& a, cudaStream_t st) {
  if (a.count == 0) return cudaSuccess;
  const int64_t tiles = (a.count + kDupItems - 1) / kDupItems;
  cudaError_t e;
  if ((e = cudaMemsetAsync(a.status, 0, sizeof(uint32_t) * tiles, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.ticket, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
  duplicate_kernel<<<static_cast<unsigned>(tiles), kDupThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_sort(const SortPlan& plan, const SortBuffers& b, int* out_buf, cudaStream_t st) {
  *out_buf = 0;
  if (plan.n <= 1 || plan.passes == 0) return cudaSuccess;
  cudaError_t e;
  if ((e = cudaMemsetAsync(b.hist, 0, sizeof(uint32_t) * kMaxPasses * kRadix, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(b.counters, 0, sizeof(uint32_t) * kMaxPasses, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(b.status, 0, sizeof(uint32_t) * kRadix * plan.tiles * plan.passes, st)) !=
      cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(onesweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(OnesweepSmem)))) != cudaSuccess)
    return e;
  int hist_blocks = static_cast<int>(std::min<int64_t>((plan.n + 4095) / 4096, 148 * 4));
  histogram_kernel<<<hist_blocks, 256, 0, st>>>(b.keys[0], plan.n, plan.passes, b.hist);
  digit_offsets_kernel<<<plan.passes, 256, 0, st>>>(b.hist, b.offsets);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int cur = 0;
  for (int p = 0; p < plan.passes; ++p) {
    OnesweepArgs o;
    o.keys_in = b.keys[cur];
    o.vals_in = b.vals[cur];
    o.keys_out = b.keys[cur ^ 1];
    o.vals_out = b.vals[cur ^ 1];
    o.n = plan.n;
    o.shift = 8 * p;
    o.digit_bits = std::min(8, plan.key_bits - 8 * p);
    o.digit_offsets = b.offsets + p * kRadix;
    o.status = b.status + static_cast<int64_t>(p) * plan.tiles * kRadix;
    o.ticket = b.counters + p;
    o.err = b.err;
    onesweep_kernel<<<static_cast<unsigned>(plan.tiles), kSortThreads, sizeof(OnesweepSmem), st>>>(o);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
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
  ranges_kernel<<<static_cast<unsigned>((n + per_block - 1) / per_block), 256, 0, st>>>(keys, n, ranges,
                                                                                       num_tiles);
  return cudaGetLastError();
}

}  // namespace gs
