// Robust photometric loss with a per-photo exposure correction (a second loss
// for the same kernels), and its gradients with respect to the image and the
// exposure parameters.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), the loss paragraph before "The chain rule, in one breath":
// err = gain C + bias - target per channel, root = sqrt(err^2 + delta^2),
// pixel loss = sum_c root - 3 delta (Charbonnier: like |err| for ordinary
// pixels, gentle for outliers), slope handed to backprop gain err / root. The
// image loss is the mean over pixels (the page reduces "to one number" without
// saying how; the mean matches the other loss).
//
// B200 design: an HBM-bound elementwise pass (24 B read, 12 B written per
// pixel) over a grid sized to the SMs, with 16-byte accesses (4 pixels per
// item) when the pixel count is a multiple of 4 and the buffers are 16-byte
// aligned; per-CTA partial sums of the loss and of the 6 exposure gradients
// in float64, reduced by the last CTA to finish in a fixed order, so the
// result is deterministic.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kCharbThreads = 256;

__global__ void __launch_bounds__(kCharbThreads) charbonnier_kernel(CharbonnierArgs a) {
  __shared__ double s_red[7][kCharbThreads / 32];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t P = a.pixels;
  const float inv = static_cast<float>(1.0 / static_cast<double>(P));
  const float d2 = a.delta * a.delta;
  float acc[7] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // sum root, dgain x3, dbias x3
  auto one = [&](int c, float x, float y) -> float {
    const float err = __fmaf_rn(a.gain[c], x, a.bias[c]) - y;
    const float root = sqrtf(__fmaf_rn(err, err, d2));
    const float slope = err / root;
    acc[0] += root;
    acc[1 + c] = __fmaf_rn(slope, x, acc[1 + c]);
    acc[4 + c] += slope;
    return a.gain[c] * slope * inv;
  };
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kCharbThreads;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kCharbThreads + tid;
  const uintptr_t bits = reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.y) |
                         reinterpret_cast<uintptr_t>(a.dx);
  if ((P & 3) == 0 && (bits & 15u) == 0) {
    // 4 pixels per item with 16-byte accesses (every channel plane then starts 16-byte aligned)
    const int64_t P4 = P >> 2;
    for (int64_t q = first; q < P4; q += stride) {
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(a.x + c * P) + q);
        const float4 y = __ldg(reinterpret_cast<const float4*>(a.y + c * P) + q);
        const float4 d = make_float4(one(c, x.x, y.x), one(c, x.y, y.y), one(c, x.z, y.z), one(c, x.w, y.w));
        if (a.dx) reinterpret_cast<float4*>(a.dx + c * P)[q] = d;
      }
    }
  } else {
    for (int64_t p = first; p < P; p += stride) {
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        const float d = one(c, __ldg(a.x + c * P + p), __ldg(a.y + c * P + p));
        if (a.dx) a.dx[c * P + p] = d;
      }
    }
  }
  double v[7];
#pragma unroll
  for (int k = 0; k < 7; ++k) {
    v[k] = acc[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
  }
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < 7; ++k) s_red[k][warp] = v[k];
  __syncthreads();
  if (tid == 0) {
    for (int k = 0; k < 7; ++k) {
      double t = 0.0;
      for (int w = 0; w < kCharbThreads / 32; ++w) t += s_red[k][w];
      a.partials[7 * blockIdx.x + k] = t;
    }
    __threadfence();
    s_last = atomicAdd(a.counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid < 7) {  // fixed-order final sums, one thread per quantity
    double t = 0.0;
    for (unsigned b = 0; b < gridDim.x; ++b) t += __ldcg(a.partials + 7 * b + tid);
    const double invP = 1.0 / static_cast<double>(P);
    a.out[tid] = tid == 0 ? t * invP - 3.0 * static_cast<double>(a.delta) : t * invP;
  }
  if (tid == 0) *a.counter = 0u;  // ready for the next call
}

}  // namespace

int charbonnier_blocks(int64_t pixels) {
  const int64_t want = (pixels + 8 * kCharbThreads - 1) / (8 * kCharbThreads);
  return static_cast<int>(want < kCharbMaxBlocks ? (want > 0 ? want : 1) : kCharbMaxBlocks);
}

cudaError_t launch_charbonnier(const CharbonnierArgs& a, cudaStream_t st) {
  charbonnier_kernel<<<charbonnier_blocks(a.pixels), kCharbThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gs
