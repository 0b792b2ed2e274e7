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
// B200 design. One CTA of 256 threads per 16x16 tile, one pixel per thread;
// each warp owns an 8x4 pixel block and walks the tile's list on its own (no
// CTA-wide barrier: a warp whose pixels are saturated stops while its
// neighbours go on). The list is consumed 32 entries at a time: lane l gathers
// entry base + l (its 48-byte screen record, prefetched one chunk ahead into
// registers), tests the record's alpha >= 1/255 box against the warp's block,
// and a ballot compacts the survivors into the warp's slice of shared memory.
// The pixel loop then visits only survivors, so a Gaussian that cannot reach
// the block costs 1/32 of a warp instruction slot instead of a full
// evaluation; the box is conservative, so results do not change.
// Per evaluated pair: alpha = min(0.99, 2^p) with the exponent-ready conic of
// the screen record (7 FP32 ops and one MUFU.EX2).
// The forward stores only the final T and n_contrib per pixel; the backward
// re-walks back to front from each pixel's last contributor, recovers T by
// dividing by (1 - alpha), and keeps one running scalar g . S (S = colour
// already composited behind) instead of three channels. Per pair it forms 9
// raw sums (w, w dx, w dy, w dx^2, w dx dy, w dy^2, dL/dc) with
// w = dL/dalpha * o exp(-e); a warp reduce-scatter (12 shuffles instead of 45)
// leaves the 9 warp totals in 9 lanes, which issue one coalesced group of 9
// float32 atomics. The conic/opacity/mean2d chain of those sums is applied
// once per Gaussian in the projection backward.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kWarps = 8;

// Warp-private slots of the surviving Gaussians of the current chunk.
struct WarpSlots {
  float2 xy[32];
  float4 q[32];    // A', B', C', log2(o)
  float4 col[32];  // r, g, b, o
  int pos[32];     // list position relative to the tile start
  uint32_t id[32];
};

// One gathered list entry: the screen record of its Gaussian.
struct Entry {
  Screen s;
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
    e.s.a = __ldg(r);
    e.s.b = __ldg(r + 1);
    e.s.c = __ldg(r + 2);
  } else {
    e.s.a = e.s.b = e.s.c = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  return e;
}

// The entry's alpha >= 1/255 box meets the pixel block [bx0, bx0+7] x [by0, by0+3].
__device__ __forceinline__ bool hits_block(const Entry& e, float bx0, float by0) {
  const float u = e.s.a.x, v = e.s.a.y, hx = e.s.c.z, hy = e.s.c.w;
  const float cx = fminf(fmaxf(u, bx0), bx0 + 7.0f);
  const float cy = fminf(fmaxf(v, by0), by0 + 3.0f);
  return e.valid && fabsf(u - cx) <= hx && fabsf(v - cy) <= hy;
}

__device__ __forceinline__ void put_slot(WarpSlots& w, int slot, const Entry& e, int pos) {
  w.xy[slot] = make_float2(e.s.a.x, e.s.a.y);
  w.q[slot] = make_float4(e.s.a.z, e.s.a.w, e.s.b.x, e.s.b.y);
  w.col[slot] = make_float4(e.s.b.z, e.s.b.w, e.s.c.x, e.s.c.y);
  w.pos[slot] = pos;
  w.id[slot] = e.gid;
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
  __shared__ WarpSlots slots[kWarps];
  const int tile = blockIdx.x;
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
    if (keep) put_slot(ws, __popc(mask & lt), cur, base + lane - beg);
    __syncwarp();
    const int cnt = __popc(mask);
    for (int k = 0; k < cnt; ++k) {
      const float2 xy = ws.xy[k];
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
        last = ws.pos[k] + 1;
        done = T < kTMin;
      }
    }
    __syncwarp();  // the slots are rewritten by the next chunk
  }
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

// Reduces v[0..8] over the warp; on return lane l (l even) holds the warp total
// of v[idx], idx = 8 b1 + 4 b2 + 2 b3 + b4 with b_k = bit k of l.
__device__ __forceinline__ float warp_reduce_scatter9(const float (&v)[9], int lane) {
  const unsigned full = 0xffffffffu;
  float w[5];
  {
    const bool up = lane & 16;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const float a0 = v[2 * i], a1 = (2 * i + 1 < 9) ? v[2 * i + 1] : 0.0f;
      const float send = up ? a0 : a1, keep = up ? a1 : a0;
      w[i] = keep + __shfl_xor_sync(full, send, 16);
    }
  }
  float x[3];
  {
    const bool up = lane & 8;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const float a0 = w[2 * i], a1 = (2 * i + 1 < 5) ? w[2 * i + 1] : 0.0f;
      const float send = up ? a0 : a1, keep = up ? a1 : a0;
      x[i] = keep + __shfl_xor_sync(full, send, 8);
    }
  }
  float y[2];
  {
    const bool up = lane & 4;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float a0 = x[2 * i], a1 = (2 * i + 1 < 3) ? x[2 * i + 1] : 0.0f;
      const float send = up ? a0 : a1, keep = up ? a1 : a0;
      y[i] = keep + __shfl_xor_sync(full, send, 4);
    }
  }
  float z;
  {
    const bool up = lane & 2;
    const float send = up ? y[0] : y[1], keep = up ? y[1] : y[0];
    z = keep + __shfl_xor_sync(full, send, 2);
  }
  return z + __shfl_xor_sync(full, z, 1);
}

template <bool kCount>
__global__ void __launch_bounds__(256) blend_backward_kernel(BlendArgs a) {
  __shared__ WarpSlots slots[kWarps];
  const int tile = blockIdx.x;
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
  // g . S with S the colour composited behind the current Gaussian; starts at T_final bg.
  float gS = T * (g0 * a.cam.bg[0] + g1 * a.cam.bg[1] + g2 * a.cam.bg[2]);
  // n_contrib comes from the caller: never walk past the tile's own list.
  int wlast = last;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wlast = max(wlast, __shfl_xor_sync(0xffffffffu, wlast, o));
  const int top = beg + max(0, min(wlast, static_cast<int>(range.y - range.x)));  // exclusive

  // Which raw sum this lane holds after the reduce-scatter.
  const int red_idx = ((lane >> 1) & 1) * 8 + ((lane >> 2) & 1) * 4 + ((lane >> 3) & 1) * 2 +
                      ((lane >> 4) & 1);
  const bool red_writer = !(lane & 1) && red_idx < 9;
  unsigned blended = 0;

  // Chunks walk down from the top; lane l takes entry hi - 1 - l, so ballot
  // order (lane order) is descending list order.
  uint32_t gid_next = load_gid(a.order, top - 1 - lane, beg, top);
  Entry nxt = load_entry(a.screen, gid_next, top - 1 - lane >= beg);
  gid_next = load_gid(a.order, top - 33 - lane, beg, top);
  for (int hi = top; hi > beg; hi -= 32) {
    const Entry cur = nxt;
    const int j_cur = hi - 1 - lane;
    nxt = load_entry(a.screen, gid_next, j_cur - 32 >= beg);
    gid_next = load_gid(a.order, j_cur - 64, beg, top);
    const bool keep = j_cur >= beg && hits_block(cur, bx0, by0);
    const unsigned mask = __ballot_sync(0xffffffffu, keep);
    if (keep) put_slot(ws, __popc(mask & lt), cur, j_cur - beg);
    __syncwarp();
    const int cnt = __popc(mask);
    for (int k = 0; k < cnt; ++k) {
      const int pos = ws.pos[k];
      const float2 xy = ws.xy[k];
      const float dx = fx - xy.x, dy = fy - xy.y;
      const float raw = fast_exp2(power2(ws.q[k], dx, dy));
      const float alpha = fminf(kAlphaMax, raw);
      const bool contrib = pos < last && alpha >= kAlphaMin;
      if (kCount && contrib) ++blended;
      if (!__any_sync(0xffffffffu, contrib)) continue;
      float v[9];
#pragma unroll
      for (int r = 0; r < 9; ++r) v[r] = 0.0f;
      if (contrib) {
        const float rcp = __fdividef(1.0f, 1.0f - alpha);
        T = T * rcp;  // transmittance in front of this Gaussian
        const float4 c = ws.col[k];
        const float gc = __fmaf_rn(g2, c.z, __fmaf_rn(g1, c.y, g0 * c.x));
        const float dalpha = __fmaf_rn(T, gc, -gS * rcp);  // dI/dalpha = T c - S / (1 - alpha)
        const float aT = alpha * T;
        gS = __fmaf_rn(gc, aT, gS);
        v[6] = g0 * aT;
        v[7] = g1 * aT;
        v[8] = g2 * aT;
        const float w = raw <= kAlphaMax ? dalpha * raw : 0.0f;  // zero through the cap
        const float wdx = w * dx, wdy = w * dy;
        v[0] = w;
        v[1] = wdx;
        v[2] = wdy;
        v[3] = wdx * dx;
        v[4] = wdx * dy;
        v[5] = wdy * dy;
      }
      const float tot = warp_reduce_scatter9(v, lane);
      if (red_writer) atomicAdd(a.sgrad + static_cast<int64_t>(ws.id[k]) * kGradStride + red_idx, tot);
    }
    __syncwarp();
  }
  if (kCount) {
    // the method's backward walk visits every entry before the pixel's last contributor
    count_pairs(a.pairs, static_cast<unsigned>(min(last, static_cast<int>(range.y - range.x))));
    count_pairs(a.pairs + 2, blended);
  }
}

}  // namespace

cudaError_t launch_blend_forward(const BlendArgs& a, cudaStream_t st) {
  const int tiles = a.cam.tiles_x * a.cam.tiles_y;
  if (tiles == 0) return cudaSuccess;
  if (a.pairs)
    blend_forward_kernel<true><<<tiles, 256, 0, st>>>(a);
  else
    blend_forward_kernel<false><<<tiles, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_blend_backward(const BlendArgs& a, cudaStream_t st) {
  const int tiles = a.cam.tiles_x * a.cam.tiles_y;
  if (tiles == 0) return cudaSuccess;
  if (a.pairs)
    blend_backward_kernel<true><<<tiles, 256, 0, st>>>(a);
  else
    blend_backward_kernel<false><<<tiles, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gs
