// Fused Adam step over one flat float32 buffer.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), Adam paragraph after "Proving the blame is right":
// m = b1 m + (1 - b1) g, v = b2 v + (1 - b2) g^2, bias-corrected m and v,
// p -= lr m_hat / (sqrt(v_hat) + eps). "Differentiable rasterisation"
// (splat-report), section "From a pixel error back to a quaternion": each
// parameter group has its own learning rate (one call per group).
//
// B200 design: purely HBM-bound, 32 B per scalar (p, g, m, v read; p, m, v and
// the zeroed g written). float4 loads/stores, grid of 148 x 8 CTAs striding
// over the buffer, bias corrections folded into two scalars on the host.
#include "adam_math.cuh"
#include "gs_kernels.cuh"

namespace gs {

namespace {

__global__ void __launch_bounds__(256) adam_vec_kernel(float4* __restrict__ p, float4* __restrict__ g,
                                                       float4* __restrict__ m, float4* __restrict__ v,
                                                       int64_t n4, AdamScalars s) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 pp = p[i], gg = g[i], mm = m[i], vv = v[i];
    adam_one(pp.x, gg.x, mm.x, vv.x, s);
    adam_one(pp.y, gg.y, mm.y, vv.y, s);
    adam_one(pp.z, gg.z, mm.z, vv.z, s);
    adam_one(pp.w, gg.w, mm.w, vv.w, s);
    p[i] = pp;
    g[i] = gg;
    m[i] = mm;
    v[i] = vv;
  }
}

__global__ void adam_scalar_kernel(float* p, float* g, float* m, float* v, int64_t n, AdamScalars s) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    adam_one(p[i], g[i], m[i], v[i], s);
}

}  // namespace

AdamScalars adam_scalars(float lr, float beta1, float beta2, float eps, int step) {
  AdamScalars s;
  const double bc1 = 1.0 - pow(static_cast<double>(beta1), step);
  const double bc2 = 1.0 - pow(static_cast<double>(beta2), step);
  s.step_size = static_cast<float>(lr / bc1);
  s.inv_sqrt_bc2 = static_cast<float>(1.0 / sqrt(bc2));
  s.beta1 = beta1;
  s.beta2 = beta2;
  s.eps = eps;
  return s;
}

cudaError_t launch_adam(float* p, float* g, float* m, float* v, int64_t count, float lr, float beta1,
                        float beta2, float eps, int step, cudaStream_t st) {
  if (count == 0) return cudaSuccess;
  const AdamScalars s = adam_scalars(lr, beta1, beta2, eps, step);
  const bool aligned = ((reinterpret_cast<uintptr_t>(p) | reinterpret_cast<uintptr_t>(g) |
                         reinterpret_cast<uintptr_t>(m) | reinterpret_cast<uintptr_t>(v)) & 15u) == 0;
  int64_t done = 0;
  if (aligned) {
    const int64_t n4 = count / 4;
    if (n4 > 0) {
      const int64_t want = (n4 + 255) / 256;
      const unsigned blocks = static_cast<unsigned>(want < 148 * 8 ? want : 148 * 8);
      adam_vec_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<float4*>(p), reinterpret_cast<float4*>(g),
                                              reinterpret_cast<float4*>(m), reinterpret_cast<float4*>(v),
                                              n4, s);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    done = n4 * 4;
  }
  const int64_t rest = count - done;
  if (rest > 0) {
    const int64_t want = (rest + 255) / 256;
    const unsigned blocks = static_cast<unsigned>(want < 148 * 8 ? want : 148 * 8);
    adam_scalar_kernel<<<blocks, 256, 0, st>>>(p + done, g + done, m + done, v + done, rest, s);
  }
  return cudaGetLastError();
}

}  // namespace gs
