// Forward and backward alpha blending over the sorted per-tile lists.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), sections "The painting itself: front-to-back alpha
// compositing" and "The clever bit: a single backward sweep through the
// blend"; "Differentiable rasterisation" (splat-report), section "The trick:
// recompute the blend state instead of storing it"; "Gaussian splatting
// training" study notes (bailiping.com), slide on alpha (cap 0.99, skip below
// 1/255, stop when nearly opaque) and slide "r is the RGB loss gradient".
//
// B200 design. One CTA of 256 threads per 16x16 tile, one pixel per thread,
// the tiles taken longest list first; each warp owns an 8x4 pixel block and
// walks the tile's list on its own (no CTA-wide barrier: a warp whose pixels
// are saturated stops while its neighbours go on). The list is consumed 32
// entries at a time: lane l gathers entry base + l (its 48-byte screen record,
// prefetched one chunk ahead into registers), tests the record's
// alpha >= 1/255 box against the warp's block, and a ballot compacts the
// survivors into the warp's slots in shared memory. The pixel loop then
// visits only survivors, so a Gaussian that cannot reach the block costs 1/32
// of a warp instruction slot instead of a full evaluation; the box is
// conservative, so results do not change.
// Per evaluated pair: alpha = min(0.99, 2^p) with the exponent-ready conic of
// the screen record (7 FP32 ops and one MUFU.EX2).
// The forward stores only the final T and n_contrib per pixel, and for each
// warp the survivors that blended at one of its pixels. The backward walks
// those back to front from each pixel's last contributor, recovers T by
// dividing by (1 - alpha), and keeps one running scalar g . S (S = colour
// already composited behind) instead of three channels. Per (Gaussian, pixel)
// it keeps two factors, w = dL/dalpha * o exp(-e) and alpha T, in a per-warp
// batch in shared memory; at the end of each half of a chunk of survivor
// slots (16 Gaussians, fewer at a walk's start) two lanes per Gaussian reduce
// its row into its 9 raw sums (w, w dx, w dy, w dx^2, w dx dy, w dy^2, dL/dc)
// and add them with float32 atomics. The conic/opacity/mean2d chain
// of those sums is applied once per Gaussian in the projection backward.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kWarps = 8;

// Warp-private slots of the surviving Gaussians of the current chunk. The
// centre, the list position and the Gaussian share one 16-byte slot, so a
// survivor's bookkeeping comes with the load of its centre.
struct WarpSlots {
  float4 xyp[32];  // u, v, list position relative to the tile start (int bits), Gaussian (uint bits)
  float4 q[32];    // A', B', C', log2(o)
  float4 col[32];  // r, g, b, o
};

__device__ __forceinline__ int slot_pos(const float4& xyp) { return __float_as_int(xyp.z); }
__device__ __forceinline__ uint32_t slot_id(const float4& xyp) { return __float_as_uint(xyp.w); }

// One gathered list entry: its Gaussian and that Gaussian's screen record.
struct Entry {
  float4 box;  // u, v, hx, hy
  float4 q;    // A', B', C', log2(o)
  float4 col;  // r, g, b, o
  uint32_t gid;
  bool valid;
};

__device__ __forceinline__ uint32_t load_gid(const uint32_t* order, int j, int lo, int hi) {
  return (j >= lo && j < hi) ? __ldg(order + j) : 0u;
}

__device__ __forceinline__ Entry load_entry(const Screen* screen, uint32_t gid, bool valid) {
  Entry e;
  e.valid = valid;
  e.gid = gid;
  if (valid) {
    const float4* r = reinterpret_cast<const float4*>(screen + gid);
    e.box = __ldg(r);
    e.q = __ldg(r + 1);
    e.col = __ldg(r + 2);
  } else {
    e.box = e.q = e.col = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  return e;
}

// The entry's alpha >= 1/255 box meets the pixel block [bx0, bx0+7] x [by0, by0+3].
__device__ __forceinline__ bool hits_block(const Entry& e, float bx0, float by0) {
  const float u = e.box.x, v = e.box.y, hx = e.box.z, hy = e.box.w;
  const float cx = fminf(fmaxf(u, bx0), bx0 + 7.0f);
  const float cy = fminf(fmaxf(v, by0), by0 + 3.0f);
  return e.valid && fabsf(u - cx) <= hx && fabsf(v - cy) <= hy;
}

__device__ __forceinline__ void put_slot(WarpSlots& w, int slot, const Entry& e, int pos) {
  w.xyp[slot] = make_float4(e.box.x, e.box.y, __int_as_float(pos), __uint_as_float(e.gid));
  w.q[slot] = e.q;
  w.col[slot] = e.col;
}

// 2^x in one MUFU instruction (flushes results below 2^-126 to 0, far under
// the 1/255 floor).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Exponent in base 2 of o exp(-e) at offset (dx, dy); identical in both passes.
__device__ __forceinline__ float power2(const float4 q, float dx, float dy) {
  const float t = __fmaf_rn(__fmul_rn(q.z, dy), dy, q.w);
  const float s = __fmaf_rn(q.x, dx, __fmul_rn(q.y, dy));
  return __fmaf_rn(s, dx, t);
}

// Adds this warp's count to *pairs (profiling builds of the kernels only).
__device__ __forceinline__ void count_pairs(unsigned long long* pairs, unsigned c) {
  unsigned long long v = c;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0 && v) atomicAdd(pairs, v);
}

template <bool kCount>
__global__ void __launch_bounds__(256) blend_forward_kernel(BlendArgs a) {
  chain_wait();
  chain_release();
  __shared__ WarpSlots slots[kWarps];
  const int tile = static_cast<int>(a.tile_order[blockIdx.x]);
  const int tx = tile % a.cam.tiles_x, ty = tile / a.cam.tiles_x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  WarpSlots& ws = slots[warp];
  int lx, ly;
  tile_pixel(threadIdx.x, lx, ly);
  const int px = tx * kTile + lx, py = ty * kTile + ly;
  const bool inside = px < a.cam.width && py < a.cam.height;
  const float fx = static_cast<float>(px), fy = static_cast<float>(py);
  const float bx0 = static_cast<float>(tx * kTile + (warp & 1) * 8);
  const float by0 = static_cast<float>(ty * kTile + (warp >> 1) * 4);
  const uint2 range = a.ranges[tile];
  const int beg = static_cast<int>(range.x), end = static_cast<int>(range.y);
  const unsigned lt = (1u << lane) - 1u;

  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int last = 0;
  bool done = !inside;
  unsigned blended = 0;
  // this warp's survivors of the box test that blend at one of its pixels, in
  // list order, for the backward
  uint2* surv = a.surv + 8LL * beg + static_cast<int64_t>(warp) * (end - beg);
  int nsurv = 0;

  // two-stage prefetch: the order entries of chunk i+2, the records of chunk i+1
  uint32_t gid_next = load_gid(a.order, beg + lane, beg, end);
  Entry nxt = load_entry(a.screen, gid_next, beg + lane < end);
  gid_next = load_gid(a.order, beg + 32 + lane, beg, end);
  for (int base = beg; base < end; base += 32) {
    if (__all_sync(0xffffffffu, done)) break;
    const Entry cur = nxt;
    nxt = load_entry(a.screen, gid_next, base + 32 + lane < end);
    gid_next = load_gid(a.order, base + 64 + lane, beg, end);
    const bool keep = hits_block(cur, bx0, by0);
    const unsigned mask = __ballot_sync(0xffffffffu, keep);
    const int slot = __popc(mask & lt);
    if (keep) put_slot(ws, slot, cur, base + lane - beg);
    __syncwarp();
    const int cnt = __popc(mask);
    unsigned blent = 0u;  // slots that blended at this pixel
    for (int k = 0; k < cnt; ++k) {
      const float4 xy = ws.xyp[k];
      const float p = power2(ws.q[k], fx - xy.x, fy - xy.y);
      const float alpha = fminf(kAlphaMax, fast_exp2(p));
      if (!done && alpha >= kAlphaMin) {
        if (kCount) ++blended;
        const float4 c = ws.col[k];
        const float w = alpha * T;
        C0 = __fmaf_rn(w, c.x, C0);
        C1 = __fmaf_rn(w, c.y, C1);
        C2 = __fmaf_rn(w, c.z, C2);
        T = T * (1.0f - alpha);
        blent |= 1u << k;
        done = T < kTMin;
      }
    }
    // The backward needs only the survivors that blended at some pixel of the
    // warp (about a fifth of the box survivors blend at none on dense scenes).
    const unsigned used = __reduce_or_sync(0xffffffffu, blent);
    const bool put = keep && ((used >> slot) & 1u);
    const unsigned pm = __ballot_sync(0xffffffffu, put);
    if (put) surv[nsurv + __popc(pm & lt)] = make_uint2(static_cast<uint32_t>(base + lane - beg), cur.gid);
    nsurv += __popc(pm);
    // the last contributor so far: this chunk's last blended slot, if any
    if (blent) last = slot_pos(ws.xyp[31 - __clz(blent)]) + 1;
    __syncwarp();  // the slots are rewritten by the next chunk
  }
  if (lane == 0) a.surv_count[tile * kWarps + warp] = static_cast<uint32_t>(nsurv);
  if (inside) {
    const int64_t hw = static_cast<int64_t>(a.cam.width) * a.cam.height;
    const int64_t pix = static_cast<int64_t>(py) * a.cam.width + px;
    a.image[pix] = __fmaf_rn(T, a.cam.bg[0], C0);
    a.image[hw + pix] = __fmaf_rn(T, a.cam.bg[1], C1);
    a.image[2 * hw + pix] = __fmaf_rn(T, a.cam.bg[2], C2);
    a.final_T[pix] = T;
    a.n_contrib[pix] = last;
  }
  if (kCount) {
    // the method's walk evaluates every list entry up to the one that saturates
    // the pixel (all of them if it never saturates); culling skips most of them
    const unsigned walked = !inside ? 0u : (done ? static_cast<unsigned>(last) : static_cast<unsigned>(end - beg));
    count_pairs(a.pairs, walked);
    count_pairs(a.pairs + 2, blended);
  }
}

// Per-warp batch of Gaussians that had a contributing pixel in the backward:
// per (Gaussian, pixel) the two per-pixel factors the nine raw sums are built
// from, w = dL/dalpha * o exp(-e) and alpha T. Rows are padded to 33 so that a
// lane per Gaussian reads without bank conflicts. A batch is one half of a
// chunk's slots, so the reduction reads each Gaussian's centre and id from its
// slot (shared-memory bandwidth limits the backward as much as issue does:
// nothing per survivor is copied into the batch but its two factors).
constexpr int kBatch = 16;
struct WarpBatch {
  float2 wa[kBatch][33];  // (w, alpha T) of Gaussian j at pixel p (lane p)
  float4 g[32];           // dL/d(pixel colour) of the warp's pixels
};

// Turns a full (or final, partial) batch into the nine raw sums of each of its
// `cnt` Gaussians and adds them to sgrad. Lane j (mod 16) owns Gaussian j; the
// two half-warps take pixel rows 0-1 and 2-3 of the 8x4 block and add their
// halves with one shuffle per sum. The six spatial sums are first formed as
// moments of w over the pixel offsets from the block centre (lx, ly in
// {-3.5..3.5} x {-1.5..1.5}, compile-time constants here) and then shifted to
// the offsets from the Gaussian's centre, dx = lx - a, dy = ly - b with
// (a, b) = centre - block centre:
//   sum w dx = Mx - a M0, sum w dx^2 = Mxx - 2a Mx + a^2 M0, and so on.
// Adds v to raw sum r of a Gaussian: a float32 atomic, or, in deterministic
// mode, an integer atomic of v in 2^-40 fixed point (integer sums do not
// depend on the order the warps arrive in, so the result is bitwise
// reproducible; |v| is clamped to 2^22, far above any screen-gradient sum).
template <bool kFixed>
__device__ __forceinline__ void add_sum(float* dst, unsigned long long* fdst, int r, float v) {
  if (kFixed) {
    const double q = fmin(fmax(static_cast<double>(v) * kFixedScale, -kFixedClamp), kFixedClamp);
    atomicAdd(fdst + r, static_cast<unsigned long long>(__double2ll_rn(q)));
  } else {
    atomicAdd(dst + r, v);
  }
}

template <bool kFixed>
__device__ __forceinline__ void flush_batch(const WarpBatch& b, int cnt, int lane, float cxb, float cyb,
                                            float2 uv, uint32_t gid, float* sgrad, unsigned long long* sgrad_fixed) {
  const int j = lane & 15, h = lane >> 4;
  float m0 = 0.f, mx = 0.f, my = 0.f, mxx = 0.f, mxy = 0.f, myy = 0.f;
  float c0 = 0.f, c1 = 0.f, c2 = 0.f;
  if (j < cnt) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int p = 16 * h + i;
      const float2 wa = b.wa[j][p];
      const float4 g = b.g[p];
      constexpr float kLx[8] = {-3.5f, -2.5f, -1.5f, -0.5f, 0.5f, 1.5f, 2.5f, 3.5f};
      const float lx = kLx[i & 7];
      const float ly = (i >> 3) ? -0.5f : -1.5f;  // this half's rows, before the 2h shift
      m0 += wa.x;
      mx = __fmaf_rn(wa.x, lx, mx);
      my = __fmaf_rn(wa.x, ly, my);
      mxx = __fmaf_rn(wa.x, lx * lx, mxx);
      mxy = __fmaf_rn(wa.x, lx * ly, mxy);
      myy = __fmaf_rn(wa.x, ly * ly, myy);
      c0 = __fmaf_rn(wa.y, g.x, c0);
      c1 = __fmaf_rn(wa.y, g.y, c1);
      c2 = __fmaf_rn(wa.y, g.z, c2);
    }
    // rows of the upper half sit 2h further down: ly -> ly + 2h
    const float sh = 2.0f * static_cast<float>(h);
    myy = __fmaf_rn(sh, __fmaf_rn(sh, m0, 2.0f * my), myy);
    mxy = __fmaf_rn(sh, mx, mxy);
    my = __fmaf_rn(sh, m0, my);
  }
  const unsigned full = 0xffffffffu;
  m0 += __shfl_xor_sync(full, m0, 16);
  mx += __shfl_xor_sync(full, mx, 16);
  my += __shfl_xor_sync(full, my, 16);
  mxx += __shfl_xor_sync(full, mxx, 16);
  mxy += __shfl_xor_sync(full, mxy, 16);
  myy += __shfl_xor_sync(full, myy, 16);
  c0 += __shfl_xor_sync(full, c0, 16);
  c1 += __shfl_xor_sync(full, c1, 16);
  c2 += __shfl_xor_sync(full, c2, 16);
  if (j < cnt) {
    const float a = uv.x - cxb, bb = uv.y - cyb;
    float* dst = sgrad + static_cast<int64_t>(gid) * kGradStride;
    unsigned long long* fdst = kFixed ? sgrad_fixed + static_cast<int64_t>(gid) * kFixedStride : nullptr;
    if (h == 0) {
      const float sy = __fmaf_rn(-bb, m0, my);
      add_sum<kFixed>(dst, fdst, 0, m0);
      add_sum<kFixed>(dst, fdst, 1, __fmaf_rn(-a, m0, mx));
      add_sum<kFixed>(dst, fdst, 2, sy);
      add_sum<kFixed>(dst, fdst, 3, __fmaf_rn(a, __fmaf_rn(a, m0, -2.0f * mx), mxx));
      add_sum<kFixed>(dst, fdst, 4, __fmaf_rn(-a, sy, __fmaf_rn(-bb, mx, mxy)));
    } else {
      add_sum<kFixed>(dst, fdst, 5, __fmaf_rn(bb, __fmaf_rn(bb, m0, -2.0f * my), myy));
      add_sum<kFixed>(dst, fdst, 6, c0);
      add_sum<kFixed>(dst, fdst, 7, c1);
      add_sum<kFixed>(dst, fdst, 8, c2);
    }
  }
}

struct BackwardSmem {
  WarpSlots slots[kWarps];
  WarpBatch batches[kWarps];
};

// Four CTAs per SM (64 registers) where that needs no spills; the
// fixed-point variant keeps three.
template <bool kCount, bool kFixed>
__global__ void __launch_bounds__(256, kFixed ? 3 : 4) blend_backward_kernel(BlendArgs a) {
  chain_wait();
  chain_release();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BackwardSmem& sm = *reinterpret_cast<BackwardSmem*>(smem_raw);
  WarpSlots* slots = sm.slots;
  WarpBatch* batches = sm.batches;
  const int tile = static_cast<int>(a.tile_order[blockIdx.x]);
  const int tx = tile % a.cam.tiles_x, ty = tile / a.cam.tiles_x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  WarpSlots& ws = slots[warp];
  WarpBatch& wb = batches[warp];
  int lx, ly;
  tile_pixel(threadIdx.x, lx, ly);
  const int px = tx * kTile + lx, py = ty * kTile + ly;
  const bool inside = px < a.cam.width && py < a.cam.height;
  const float fx = static_cast<float>(px), fy = static_cast<float>(py);
  const float bx0 = static_cast<float>(tx * kTile + (warp & 1) * 8);
  const float by0 = static_cast<float>(ty * kTile + (warp >> 1) * 4);
  const uint2 range = a.ranges[tile];
  const int beg = static_cast<int>(range.x);
  const unsigned lt = (1u << lane) - 1u;

  const int64_t hw = static_cast<int64_t>(a.cam.width) * a.cam.height;
  const int64_t pix = static_cast<int64_t>(py) * a.cam.width + px;
  float T = 0.0f, g0 = 0.0f, g1 = 0.0f, g2 = 0.0f;
  int last = 0;
  if (inside) {
    T = a.final_T[pix];
    last = a.n_contrib[pix];
    g0 = a.dimage[pix];
    g1 = a.dimage[hw + pix];
    g2 = a.dimage[2 * hw + pix];
  }
  wb.g[lane] = make_float4(g0, g1, g2, 0.0f);
  // g . S with S the colour composited behind the current Gaussian; starts at T_final bg.
  float gS = T * (g0 * a.cam.bg[0] + g1 * a.cam.bg[1] + g2 * a.cam.bg[2]);
  // n_contrib comes from the caller: never walk past the tile's own list.
  int wlast = last;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wlast = max(wlast, __shfl_xor_sync(0xffffffffu, wlast, o));
  const int top = beg + max(0, min(wlast, static_cast<int>(range.y - range.x)));  // exclusive
  unsigned blended = 0;

  // The forward stored this warp's survivors of the box test that blend at one
  // of its pixels (list position, Gaussian) in list order; walk them from the
  // last one down. Lane l takes survivor hi - 1 - l, so ballot order (lane
  // order) is descending list order; survivors at or past the warp's last
  // contributor are dropped.
  const int end = static_cast<int>(range.y);
  const uint2* surv = a.surv + 8LL * beg + static_cast<int64_t>(warp) * (end - beg);
  const int nsurv = min(static_cast<int>(a.surv_count[tile * kWarps + warp]), end - beg);
  const int toprel = top - beg;
  uint2 sv_next = nsurv - 1 - lane >= 0 ? surv[nsurv - 1 - lane] : make_uint2(0u, 0u);
  Entry nxt = load_entry(a.screen, sv_next.y, nsurv - 1 - lane >= 0);
  int pos_next = static_cast<int>(sv_next.x);
  sv_next = nsurv - 33 - lane >= 0 ? surv[nsurv - 33 - lane] : make_uint2(0u, 0u);
  for (int hi = nsurv; hi > 0; hi -= 32) {
    const Entry cur = nxt;
    const int pos_cur = pos_next;
    const int j_cur = hi - 1 - lane;
    nxt = load_entry(a.screen, sv_next.y, j_cur - 32 >= 0);
    pos_next = static_cast<int>(sv_next.x);
    sv_next = j_cur - 64 >= 0 ? surv[j_cur - 64] : make_uint2(0u, 0u);
    const bool keep = j_cur >= 0 && pos_cur < toprel;
    const unsigned mask = __ballot_sync(0xffffffffu, keep);
    if (keep) put_slot(ws, __popc(mask & lt), cur, pos_cur);
    __syncwarp();
    const int cnt = __popc(mask);
    for (int k = 0; k < cnt; ++k) {
      const float4 xy = ws.xyp[k];
      const int pos = slot_pos(xy);
      const float dx = fx - xy.x, dy = fy - xy.y;
      const float raw = fast_exp2(power2(ws.q[k], dx, dy));
      const float alpha = fminf(kAlphaMax, raw);
      const bool contrib = pos < last && alpha >= kAlphaMin;
      if (kCount && contrib) ++blended;
      // Every stored survivor blended at some pixel of the warp in the forward,
      // with the same alpha and before that pixel's last contributor, so some
      // lane contributes here: no vote is needed to skip it (and a survivor
      // with none would only add zeros).
      // Every lane computes the update (the warp runs it anyway, as some lane
      // contributes) and keeps it only where its pixel contributes: no branch,
      // so the next survivor's loads and exponential can start early.
      const float rcp = __fdividef(1.0f, 1.0f - alpha);
      const float Tf = T * rcp;  // transmittance in front of this Gaussian
      const float4 c = ws.col[k];
      const float gc = __fmaf_rn(g2, c.z, __fmaf_rn(g1, c.y, g0 * c.x));
      const float dalpha = __fmaf_rn(Tf, gc, -gS * rcp);  // dI/dalpha = T c - S / (1 - alpha)
      const float aTf = alpha * Tf;
      const float aT = contrib ? aTf : 0.0f;
      const float w = (contrib && raw <= kAlphaMax) ? dalpha * raw : 0.0f;  // zero through the cap
      T = contrib ? Tf : T;
      gS = __fmaf_rn(gc, aT, gS);
      // A batch is slots 16 h .. 16 h + 15 of the chunk (fewer in its last
      // one), so its Gaussians' centres and ids are still in the slots when it
      // is reduced.
      const int row = k & (kBatch - 1);
      wb.wa[row][lane] = make_float2(w, aT);
      if (row == kBatch - 1 || k == cnt - 1) {
        __syncwarp();
        const float4 bxy = ws.xyp[k - row + (lane & (kBatch - 1))];
        flush_batch<kFixed>(wb, row + 1, lane, bx0 + 3.5f, by0 + 1.5f, make_float2(bxy.x, bxy.y), slot_id(bxy),
                            a.sgrad, a.sgrad_fixed);
        __syncwarp();
      }
    }
    __syncwarp();  // the slots are rewritten by the next chunk
  }
  if (kCount) {
    // the method's backward walk visits every entry before the pixel's last contributor
    count_pairs(a.pairs, static_cast<unsigned>(min(last, static_cast<int>(range.y - range.x))));
    count_pairs(a.pairs + 2, blended);
  }
}

// Deterministic mode: the fixed-point sums back to float32 raw sums.
__global__ void decode_fixed_kernel(const unsigned long long* fixed, int64_t n, float* sgrad) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const unsigned long long* f = fixed + i * kFixedStride;
  float* o = sgrad + i * kGradStride;
#pragma unroll
  for (int r = 0; r < 9; ++r)
    o[r] = static_cast<float>(static_cast<double>(static_cast<long long>(f[r])) / kFixedScale);
#pragma unroll
  for (int r = 9; r < kGradStride; ++r) o[r] = 0.0f;
}

}  // namespace

cudaError_t launch_decode_fixed(const unsigned long long* fixed, int64_t n, float* sgrad, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  decode_fixed_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(fixed, n, sgrad);
  return cudaGetLastError();
}

cudaError_t launch_blend_forward(const BlendArgs& a, cudaStream_t st) {
  const int tiles = a.cam.tiles_x * a.cam.tiles_y;
  if (tiles == 0) return cudaSuccess;
  return a.pairs ? launch_chained(blend_forward_kernel<true>, dim3(tiles), dim3(256), 0, st, a)
                 : launch_chained(blend_forward_kernel<false>, dim3(tiles), dim3(256), 0, st, a);
}

template <bool kCount, bool kFixed>
cudaError_t launch_backward_variant(const BlendArgs& a, int tiles, cudaStream_t st) {
  const int smem = static_cast<int>(sizeof(BackwardSmem));
  cudaError_t e = cudaFuncSetAttribute(blend_backward_kernel<kCount, kFixed>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_chained(blend_backward_kernel<kCount, kFixed>, dim3(tiles), dim3(256), smem, st, a);
}

cudaError_t launch_blend_backward(const BlendArgs& a, cudaStream_t st) {
  const int tiles = a.cam.tiles_x * a.cam.tiles_y;
  if (tiles == 0) return cudaSuccess;
  if (a.pairs)
    return a.sgrad_fixed ? launch_backward_variant<true, true>(a, tiles, st)
                         : launch_backward_variant<true, false>(a, tiles, st);
  return a.sgrad_fixed ? launch_backward_variant<false, true>(a, tiles, st)
                       : launch_backward_variant<false, false>(a, tiles, st);
}

}  // namespace gs
