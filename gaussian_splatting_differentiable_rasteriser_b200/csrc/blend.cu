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
// each warp an 8x4 pixel block (compact blocks let the backward skip whole
// warps a small Gaussian does not reach). The tile's sorted Gaussians are
// gathered from the 48-byte screen records in batches of 256 into shared
// memory, already rescaled for the exponent: alpha = min(0.99, 2^p) with
//     p = A' dx^2 + B' dx dy + C' dy^2 + log2(o),
//     A' = -A log2(e) / 2, B' = -B log2(e), C' = -C log2(e) / 2,
// so each (pixel, Gaussian) pair costs 7 FP32 ops, one MUFU.EX2 and a min.
// The forward stops a CTA when every pixel is saturated (syncthreads_count).
// The forward stores only the final T and n_contrib per pixel; the backward
// re-walks back to front from each pixel's last contributor, recovers T by
// dividing by (1 - alpha), and keeps a single running scalar g . S (S = colour
// already composited behind) instead of the three channels. Per pair it
// produces 9 raw sums (w, w dx, w dy, w dx^2, w dx dy, w dy^2, dL/dc) with
// w = dL/dalpha * o exp(-e); a warp reduce-scatter (12 shuffles instead of 45)
// leaves the 9 warp totals in 9 lanes, which issue one coalesced group of 9
// float32 atomics. The conic/opacity/mean2d chain of those sums is applied once
// per Gaussian in the projection backward.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kBatch = 256;

// Shared-memory copy of one batch of Gaussians.
struct BlendSmem {
  float2 xy[kBatch];
  float4 q[kBatch];    // A', B', C', log2(o)
  float4 col[kBatch];  // r, g, b, o
  float4 box[kBatch];  // x_lo, x_hi, y_lo, y_hi of the alpha >= 1/255 region
  uint32_t id[kBatch];
};

__device__ __forceinline__ void stage(BlendSmem& s, int slot, uint32_t gid, const Screen* screen) {
  const Screen g = screen[gid];
  const float u = g.a.x, v = g.a.y, A = g.a.z, B = g.a.w, C = g.b.x, o = g.b.y;
  s.xy[slot] = make_float2(u, v);
  s.q[slot] = make_float4(__fmul_rn(-0.5f * kLog2e, A), __fmul_rn(-kLog2e, B),
                          __fmul_rn(-0.5f * kLog2e, C), log2f(o));
  s.col[slot] = make_float4(g.b.z, g.b.w, g.c.x, o);
  // o exp(-e) >= 1/255 exactly when e <= E = ln(255 o); the ellipse e <= E has the
  // axis-aligned half-widths sqrt(2 E Sigma'_xx), sqrt(2 E Sigma'_yy), with
  // Sigma' = conic^-1. The box is widened by 0.1% + 0.02 px so that float32
  // rounding of the per-pixel alpha can never pass the floor outside it: a warp
  // whose pixels all lie outside skips the Gaussian with unchanged results.
  const float E = logf(255.0f * o);
  float4 box = make_float4(1.0f, -1.0f, 1.0f, -1.0f);  // empty
  const float det = A * C - B * B;
  if (E > 0.0f && det > 0.0f) {
    const float hx = sqrtf(2.0f * E * C / det) * 1.001f + 0.02f;
    const float hy = sqrtf(2.0f * E * A / det) * 1.001f + 0.02f;
    box = make_float4(u - hx, u + hx, v - hy, v + hy);
  }
  s.box[slot] = box;
  s.id[slot] = gid;
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

// True when the Gaussian's alpha >= 1/255 box misses the warp's 8x4 pixel block.
__device__ __forceinline__ bool misses_block(const float4 box, float bx0, float bx1, float by0,
                                             float by1) {
  return box.y < bx0 || box.x > bx1 || box.w < by0 || box.z > by1;
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
  __shared__ BlendSmem sm;
  const int tile = blockIdx.x;
  const int tx = tile % a.cam.tiles_x, ty = tile / a.cam.tiles_x;
  int lx, ly;
  tile_pixel(threadIdx.x, lx, ly);
  const int px = tx * kTile + lx, py = ty * kTile + ly;
  const bool inside = px < a.cam.width && py < a.cam.height;
  const uint2 range = a.ranges[tile];
  const int n = static_cast<int>(range.y - range.x);
  const float fx = static_cast<float>(px), fy = static_cast<float>(py);

  // this warp's 8x4 pixel block
  const float bx0 = static_cast<float>(tx * kTile + ((threadIdx.x >> 5) & 1) * 8);
  const float by0 = static_cast<float>(ty * kTile + (threadIdx.x >> 6) * 4);
  const float bx1 = bx0 + 7.0f, by1 = by0 + 3.0f;

  float T = 1.0f, C0 = 0.0f, C1 = 0.0f, C2 = 0.0f;
  int last = 0;
  bool done = !inside;
  unsigned evals = 0;
  for (int b = 0; b < n; b += kBatch) {
    if (__syncthreads_count(!done) == 0) break;
    const int k = b + threadIdx.x;
    if (k < n) stage(sm, threadIdx.x, a.order[range.x + k], a.screen);
    __syncthreads();
    const int cnt = min(kBatch, n - b);
    if (__all_sync(0xffffffffu, done)) continue;  // this warp is saturated
    for (int j = 0; j < cnt; ++j) {
      if ((j & 31) == 31 && __all_sync(0xffffffffu, done)) break;
      if (misses_block(sm.box[j], bx0, bx1, by0, by1)) continue;
      if (kCount) evals += !done;
      const float2 xy = sm.xy[j];
      const float p = power2(sm.q[j], fx - xy.x, fy - xy.y);
      const float alpha = fminf(kAlphaMax, fast_exp2(p));
      if (!done && alpha >= kAlphaMin) {
        const float4 c = sm.col[j];
        const float w = alpha * T;
        C0 = __fmaf_rn(w, c.x, C0);
        C1 = __fmaf_rn(w, c.y, C1);
        C2 = __fmaf_rn(w, c.z, C2);
        T = T * (1.0f - alpha);
        last = b + j + 1;
        done = T < kTMin;
      }
    }
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
  if (kCount) count_pairs(a.pairs, evals);
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
  __shared__ BlendSmem sm;
  __shared__ int s_max_last;
  const int tile = blockIdx.x;
  const int tx = tile % a.cam.tiles_x, ty = tile / a.cam.tiles_x;
  const int lane = threadIdx.x & 31;
  int lx, ly;
  tile_pixel(threadIdx.x, lx, ly);
  const int px = tx * kTile + lx, py = ty * kTile + ly;
  const bool inside = px < a.cam.width && py < a.cam.height;
  const uint2 range = a.ranges[tile];
  const float fx = static_cast<float>(px), fy = static_cast<float>(py);

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

  if (threadIdx.x == 0) s_max_last = 0;
  __syncthreads();
  int wmax = last;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wmax = max(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
  if (lane == 0) atomicMax(&s_max_last, wmax);
  __syncthreads();
  // n_contrib comes from the caller: never walk past the tile's own list.
  const int max_last = min(s_max_last, static_cast<int>(range.y - range.x));

  const float bx0 = static_cast<float>(tx * kTile + ((threadIdx.x >> 5) & 1) * 8);
  const float by0 = static_cast<float>(ty * kTile + (threadIdx.x >> 6) * 4);
  const float bx1 = bx0 + 7.0f, by1 = by0 + 3.0f;
  const int warp_last = wmax;  // no lane of this warp blends anything at or after it

  // Which raw sum this lane holds after the reduce-scatter.
  const int red_idx = ((lane >> 1) & 1) * 8 + ((lane >> 2) & 1) * 4 + ((lane >> 3) & 1) * 2 +
                      ((lane >> 4) & 1);
  const bool red_writer = !(lane & 1) && red_idx < 9;
  unsigned evals = 0;

  for (int end = max_last; end > 0; end -= kBatch) {
    const int start = max(0, end - kBatch);
    __syncthreads();  // the previous batch is no longer read
    const int k = start + threadIdx.x;
    if (k < end) stage(sm, threadIdx.x, a.order[range.x + k], a.screen);
    __syncthreads();
    for (int j = min(end, warp_last) - 1; j >= start; --j) {
      const int slot = j - start;
      if (misses_block(sm.box[slot], bx0, bx1, by0, by1)) continue;
      const float2 xy = sm.xy[slot];
      const float dx = fx - xy.x, dy = fy - xy.y;
      const float raw = fast_exp2(power2(sm.q[slot], dx, dy));
      const float alpha = fminf(kAlphaMax, raw);
      const bool contrib = j < last && alpha >= kAlphaMin;
      if (kCount && j < last) ++evals;
      if (!__any_sync(0xffffffffu, contrib)) continue;
      float v[9];
#pragma unroll
      for (int r = 0; r < 9; ++r) v[r] = 0.0f;
      if (contrib) {
        const float rcp = __fdividef(1.0f, 1.0f - alpha);
        T = T * rcp;  // transmittance in front of this Gaussian
        const float4 c = sm.col[slot];
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
      if (red_writer) atomicAdd(a.sgrad + static_cast<int64_t>(sm.id[slot]) * kGradStride + red_idx, tot);
    }
  }
  if (kCount) count_pairs(a.pairs, evals);
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
