// Projection backward: per-Gaussian screen-space gradient -> stored parameters.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), sections "From a pixel's blame to the oval's shape and
// place", "The covariance chain: oval -> 3D ellipsoid -> size & tilt" and
// "Where the position gradient comes from", and the spherical-harmonics
// backward (dL/dsh_k = dL/dcolour * Y_k, plus the view-direction term into the
// position); "Gaussian splatting training" study notes (bailiping.com), slide
// "J is the 2 x 3 Jacobian of perspective projection" (the position derivative
// includes the path through J, not only the projected mean).
//
// Chain, per Gaussian (float32):
//   raw blend sums -> dL/d(mean2d, A, B, C, opacity)
//   conic K = V'^-1:        dL/dV' = -K G_K K   (G_K with the B gradient halved)
//   V' = T Sigma T^T + 0.3I: dL/dSigma = T^T G_V T,   dL/dT = 2 G_V T Sigma
//   T = J W:                dL/dJ = dL/dT W^T -> dL/d(X, Y, Z) (1/Z, 1/Z^2 terms)
//   mean2d(X, Y, Z)         -> dL/d(X, Y, Z);   dL/dp = W^T dL/dp_c
//   Sigma = M M^T:          dL/dM = 2 dL/dSigma M,  M = R(q^) diag(s)
//   dL/ds_j = sum_i dL/dM_ij R_ij (times s for the log-scale), dL/dR = dL/dM diag(s)
//   R(q^) -> dL/dq^, then dL/dq = (dL/dq^ - q^ <q^, dL/dq^>) / |q|
//   colour: dL/dsh_k = dL/dc Y_k, dL/dv = sum dL/dc sh_k grad Y_k,
//           dL/dp += (dL/dv - v <v, dL/dv>) / |p - campos|
// The result is ADDED to the caller's gradient buffers (coalesced planar RMW),
// or, in the fused variant, added to them and consumed by the Adam step of
// every parameter group in the same pass (the gradient never makes a separate
// round trip through HBM).
#include "adam_math.cuh"
#include "adam_stream.cuh"
#include "gs_kernels.cuh"
#include "projection_grad.cuh"
#include "sh.cuh"

namespace gs {

namespace {

// Density-control statistics of a Gaussian this view touched: the norm of
// dL/dmean2d and one more view (one thread per Gaussian: no atomics needed).
template <bool kStats>
__device__ __forceinline__ void add_densify_stats(const PreprocessBwdArgs& a, int64_t i, const GaussGrad& g) {
  if (kStats) {
    a.stat_accum[i] += sqrtf(g.du * g.du + g.dv * g.dv);
    a.stat_count[i] += 1u;
  }
}

// Backward that ADDS the gradient into the caller's buffers.
template <int kDeg, bool kStats, bool kMip>
__global__ void __launch_bounds__(256) preprocess_backward_kernel(PreprocessBwdArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= a.n || a.touched[i] == 0) return;
  const int64_t np = a.n_pad;
  GaussGrad g;
  geometry_grad<false, kMip>(a, i, g);
  add_densify_stats<kStats>(a, i, g);
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
  float Yk[16];
  sh_basis(kDeg, g.vx, g.vy, g.vz, Yk);
  float wsum[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) wsum[k] = 0.f;
#pragma unroll
  for (int ch = 0; ch < 3; ++ch) {
    if (g.drgb[ch] == 0.f) continue;
    const float* shc = a.sh + static_cast<int64_t>(ch) * a.sh_k * np + i;
    float* gsh = a.g_sh + static_cast<int64_t>(ch) * a.sh_k * np + i;
#pragma unroll
    for (int k = 0; k < nk; ++k) {
      const int64_t o = static_cast<int64_t>(k) * np;
      gsh[o] = __fmaf_rn(g.drgb[ch], Yk[k], gsh[o]);
      wsum[k] = __fmaf_rn(g.drgb[ch], shc[o], wsum[k]);
    }
  }
  add_view_dir_term<kDeg>(g, wsum);
#pragma unroll
  for (int c = 0; c < 3; ++c) a.g_means[c * np + i] += g.dp[c];
#pragma unroll
  for (int c = 0; c < 3; ++c) a.g_log_scales[c * np + i] += g.dls[c];
#pragma unroll
  for (int c = 0; c < 4; ++c) a.g_quats[c * np + i] += g.dq[c];
  a.g_opacity_logits[i] += g.dlogit;
}

// The same backward fused with the Adam step of every group, over all n_pad
// Gaussians (Adam is dense: invisible Gaussians still move by their moments).
// Per scalar: g = accumulated gradient + this view's gradient, then the update
// of adam_one; the gradient buffer is left zeroed. Bit-identical to the
// accumulate kernel followed by the standalone Adam kernel.
//
// Compute, then stream: a CTA owns 128 consecutive Gaussians. Phase 1 (one
// thread per Gaussian) computes the view gradient of the 11 geometric scalars
// and what the 48 SH gradients need (masked dL/dcolour and Y_k) into shared
// memory, while the first rounds of phase 2's loads are already in flight.
// Phase 2 streams Adam over the CTA's 59 planes x 128 Gaussians through
// per-thread cp.async stages (adam_stream.cuh); the kernel is bound by HBM,
// not by math.
constexpr int kFusedBlock = kStreamBlock;
constexpr int kGeomPlanes = kStreamGeom;

struct FusedSmem {
  float geom[kGeomPlanes][kFusedBlock];  // view gradient of the geometric scalars
  float drgb[3][kFusedBlock];            // masked dL/dcolour (0 when invisible)
  float Y[16][kFusedBlock];              // SH basis at the view direction
};

// kAccum: the caller's gradient buffer holds an accumulated gradient, which is
// added and then zeroed; without it the update uses this view's gradient alone
// and no gradient buffer is read or written (24 instead of 32 bytes per scalar).
template <int kDeg, bool kAccum, bool kStats, bool kMip>
__global__ void __launch_bounds__(kFusedBlock) preprocess_backward_adam_kernel(PreprocessBwdArgs a,
                                                                              FusedAdamArgs f) {
  chain_wait();
  chain_release();
  __shared__ __align__(16) FusedSmem sm;
  const int t = threadIdx.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kFusedBlock;
  const int64_t np = a.n_pad;
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
  // The first rounds of the Adam stream are in flight while phase 1 runs.
  extern __shared__ __align__(16) float4 stage[];
  const int planes = kGeomPlanes + 3 * a.sh_k;
  const int cols = stream_cols(i0, np);
  adam_stream_prologue<kAccum>(f, np, i0, cols, planes, a.sh_k, nk, stage);

  // Phase 1: this view's gradient of Gaussian i0 + t.
  {
    const int64_t i = i0 + t;
    const bool visible = i < a.n && a.touched[i] != 0;
    if (visible) {
      GaussGrad g;
      geometry_grad<false, kMip>(a, i, g);
      add_densify_stats<kStats>(a, i, g);
      float Yk[16];
      sh_basis(kDeg, g.vx, g.vy, g.vz, Yk);
      float wsum[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) wsum[k] = 0.f;
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) {
        if (g.drgb[ch] == 0.f) continue;
        const float* shc = a.sh + static_cast<int64_t>(ch) * a.sh_k * np + i;
#pragma unroll
        for (int k = 0; k < nk; ++k)
          wsum[k] = __fmaf_rn(g.drgb[ch], shc[static_cast<int64_t>(k) * np], wsum[k]);
      }
      add_view_dir_term<kDeg>(g, wsum);
      const float geom[kGeomPlanes] = {g.dp[0], g.dp[1], g.dp[2], g.dls[0], g.dls[1], g.dls[2],
                                       g.dq[0], g.dq[1], g.dq[2], g.dq[3], g.dlogit};
#pragma unroll
      for (int j = 0; j < kGeomPlanes; ++j) sm.geom[j][t] = geom[j];
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) sm.drgb[ch][t] = g.drgb[ch];
#pragma unroll
      for (int k = 0; k < 16; ++k) sm.Y[k][t] = k < nk ? Yk[k] : 0.f;
    } else {
#pragma unroll
      for (int j = 0; j < kGeomPlanes; ++j) sm.geom[j][t] = 0.f;
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) sm.drgb[ch][t] = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) sm.Y[k][t] = 0.f;
    }
  }
  __syncthreads();

  // Phase 2: Adam over the CTA's planes; the view gradient adds to the
  // accumulated one (zero without a gradient buffer).
  auto grad = [&](int pl, const PlaneInfo& info, int col, float4 g) {
    if (pl < kGeomPlanes) {
      const float4 d = reinterpret_cast<const float4*>(sm.geom[pl])[col];
      return make_float4(__fadd_rn(g.x, d.x), __fadd_rn(g.y, d.y), __fadd_rn(g.z, d.z), __fadd_rn(g.w, d.w));
    }
    if (info.k >= 0) {
      const float4 dc = reinterpret_cast<const float4*>(sm.drgb[info.ch])[col];
      const float4 y = reinterpret_cast<const float4*>(sm.Y[info.k])[col];
      return make_float4(dc.x != 0.f ? __fmaf_rn(dc.x, y.x, g.x) : g.x, dc.y != 0.f ? __fmaf_rn(dc.y, y.y, g.y) : g.y,
                         dc.z != 0.f ? __fmaf_rn(dc.z, y.z, g.z) : g.z, dc.w != 0.f ? __fmaf_rn(dc.w, y.w, g.w) : g.w);
    }
    return g;
  };
  adam_stream<kAccum>(f, np, i0, cols, planes, a.sh_k, nk, stage, grad);
}

// Natural screen-space gradient from the raw sums (for stage checks).
__global__ void screen_grads_kernel(const Screen* screen, const float* sgrad, int64_t n, float* out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float* r = sgrad + i * kGradStride;
  const Screen s = screen[i];
  const float A = conic_A(s), B = conic_B(s), C = conic_C(s), o = screen_opacity(s);
  float* d = out + i * 9;
  d[0] = A * r[1] + B * r[2];
  d[1] = B * r[1] + C * r[2];
  d[2] = -0.5f * r[3];
  d[3] = -r[4];
  d[4] = -0.5f * r[5];
  d[5] = o > 0.f ? r[0] / o : 0.f;
  d[6] = r[6];
  d[7] = r[7];
  d[8] = r[8];
}

}  // namespace

// The kernels are instantiated per active SH degree and per option (an
// accumulated gradient buffer, density statistics), so the default path
// carries no runtime test of either.
template <int kDeg, bool kMip>
cudaError_t launch_bwd_mip(const PreprocessBwdArgs& a, unsigned grid, cudaStream_t st) {
  if (a.stat_accum)
    preprocess_backward_kernel<kDeg, true, kMip><<<grid, 256, 0, st>>>(a);
  else
    preprocess_backward_kernel<kDeg, false, kMip><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <int kDeg>
cudaError_t launch_bwd_deg(const PreprocessBwdArgs& a, unsigned grid, cudaStream_t st) {
  return a.mip_comp ? launch_bwd_mip<kDeg, true>(a, grid, st) : launch_bwd_mip<kDeg, false>(a, grid, st);
}

template <int kDeg, bool kAccum, bool kStats, bool kMip>
cudaError_t launch_fused_mip(const PreprocessBwdArgs& a, const FusedAdamArgs& f, unsigned grid, cudaStream_t st) {
  const int smem = stage_bytes<kAccum>();  // the Adam stream's stage buffers
  cudaError_t e = cudaFuncSetAttribute(preprocess_backward_adam_kernel<kDeg, kAccum, kStats, kMip>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_chained(preprocess_backward_adam_kernel<kDeg, kAccum, kStats, kMip>, dim3(grid), dim3(kFusedBlock),
                        smem, st, a, f);
}

template <int kDeg, bool kAccum, bool kStats>
cudaError_t launch_fused_variant(const PreprocessBwdArgs& a, const FusedAdamArgs& f, unsigned grid, cudaStream_t st) {
  return a.mip_comp ? launch_fused_mip<kDeg, kAccum, kStats, true>(a, f, grid, st)
                    : launch_fused_mip<kDeg, kAccum, kStats, false>(a, f, grid, st);
}

template <int kDeg>
cudaError_t launch_fused_deg(const PreprocessBwdArgs& a, const FusedAdamArgs& f, unsigned grid, cudaStream_t st) {
  const bool accum = f.g[0] != nullptr, stats = a.stat_accum != nullptr;
  if (accum && stats) return launch_fused_variant<kDeg, true, true>(a, f, grid, st);
  if (accum) return launch_fused_variant<kDeg, true, false>(a, f, grid, st);
  if (stats) return launch_fused_variant<kDeg, false, true>(a, f, grid, st);
  return launch_fused_variant<kDeg, false, false>(a, f, grid, st);
}

cudaError_t launch_preprocess_backward(const PreprocessBwdArgs& a, cudaStream_t st) {
  if (a.n == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((a.n + 255) / 256);
  switch (a.active_degree) {
    case 0: return launch_bwd_deg<0>(a, grid, st);
    case 1: return launch_bwd_deg<1>(a, grid, st);
    case 2: return launch_bwd_deg<2>(a, grid, st);
    default: return launch_bwd_deg<3>(a, grid, st);
  }
}

cudaError_t launch_preprocess_backward_adam(const PreprocessBwdArgs& a, const FusedAdamArgs& f,
                                           cudaStream_t st) {
  if (a.n_pad == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((a.n_pad + kFusedBlock - 1) / kFusedBlock);
  switch (a.active_degree) {
    case 0: return launch_fused_deg<0>(a, f, grid, st);
    case 1: return launch_fused_deg<1>(a, f, grid, st);
    case 2: return launch_fused_deg<2>(a, f, grid, st);
    default: return launch_fused_deg<3>(a, f, grid, st);
  }
}

cudaError_t launch_screen_grads(const Screen* screen, const float* sgrad, int64_t n, float* out,
                                cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  screen_grads_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(screen, sgrad, n, out);
  return cudaGetLastError();
}

}  // namespace gs
