// Data-parallel update from the ranks' screen-space sums, fused with Adam.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), section "Per step" (one photo per step; with one photo per
// rank the batch gradient is the mean of the ranks' gradients), the covariance
// and position chains of "The covariance chain: oval -> 3D ellipsoid -> size &
// tilt" and "Where the position gradient comes from", and the Adam paragraph
// after "Proving the blame is right".
//
// After every rank's blend backward, rank k owns a contiguous range of
// Gaussians. For each of its Gaussians this kernel reads every rank's view of
// it - the screen record, the raw screen-gradient sums, the touched and clamp
// flags and that rank's camera, about 100 B from peer memory instead of the
// 236 B of a parameter gradient - runs the projection backward of each view,
// sums the parameter gradients in rank order and scales the sum (the batch
// mean), applies Adam to the Gaussian's 59 scalars and stores the updated
// parameters into every other rank's parameter buffer. No gradient buffer is
// written anywhere. The per-view gradients are formed by the same per-Gaussian
// algebra as the separate projection backward, and summed and scaled in the
// same order as gs_adam_step_reduce sums whole gradient buffers, so the result
// equals the gradient exchange's up to float32 rounding (the compiler may
// contract a multiply-add differently in each kernel). Every replica ends with
// the same bits: each Gaussian is updated by one kernel and copied. Plain loads
// and stores only (no multicast); the kernel waits on nothing: the caller
// orders it after every rank's blend backward and before any rank's next
// forward. Five CTAs of 128 per SM (96 registers, 43 KB of shared memory).
#include "adam_math.cuh"
#include "adam_stream.cuh"
#include "gs_kernels.cuh"
#include "projection_grad.cuh"
#include "sh.cuh"

namespace gs {

namespace {

constexpr int kViewsBlock = kStreamBlock;
constexpr int kViewsGeom = kStreamGeom;

struct ViewsSmem {
  float geom[kViewsGeom][kViewsBlock];  // summed, scaled gradient of the geometric scalars
  float shg[48][kViewsBlock];           // summed, scaled gradient of the active SH coefficients
  CamArgs cam[kMaxRanks];
};

template <int kDeg, bool kMip>
__global__ void __launch_bounds__(kViewsBlock, 5) views_backward_adam_kernel(ViewsAdamArgs a) {
  chain_wait();
  chain_release();
  __shared__ __align__(16) ViewsSmem sm;
  extern __shared__ __align__(16) float4 stage[];
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
  const int t = threadIdx.x;
  const int64_t np = a.base.n_pad;
  const int64_t i0 = a.g_lo + static_cast<int64_t>(blockIdx.x) * kViewsBlock;
  const int64_t i = i0 + t;
  const int planes = kViewsGeom + 3 * a.base.sh_k;
  const int cols = stream_cols(i0, a.g_hi);  // g_hi % 4 == 0
  // The first rounds of the Adam stream are in flight while phase 1 runs.
  adam_stream_prologue<false>(a.f, np, i0, cols, planes, a.base.sh_k, nk, stage);
  // every view's camera, read once per CTA from that rank's memory
  constexpr int kCamWords = static_cast<int>(sizeof(CamArgs) / 4);
  static_assert(sizeof(CamArgs) % 4 == 0, "camera record");
  for (int k = t; k < a.n_views * kCamWords; k += kViewsBlock)
    reinterpret_cast<uint32_t*>(sm.cam)[k] =
        reinterpret_cast<const uint32_t*>(a.views[k / kCamWords].cam)[k % kCamWords];
#pragma unroll
  for (int c = 0; c < 3 * nk; ++c) sm.shg[c][t] = 0.f;
  __syncthreads();

  // Phase 1: this Gaussian's gradient, view by view in rank order.
  float geom[kViewsGeom];
#pragma unroll
  for (int j = 0; j < kViewsGeom; ++j) geom[j] = 0.f;
  if (i < a.g_hi && i < a.base.n) {
    for (int r = 0; r < a.n_views; ++r) {
      const ViewArgs& vw = a.views[r];
      if (vw.touched[i] == 0u) continue;
      PreprocessBwdArgs pb = a.base;
      pb.cam = sm.cam[r];
      pb.screen = vw.screen;
      pb.sgrad = vw.sgrad;
      pb.touched = vw.touched;
      pb.clamped = vw.clamped;
      GaussGrad g;
      geometry_grad<false, kMip>(pb, i, g);
      float Yk[16];
      sh_basis(kDeg, g.vx, g.vy, g.vz, Yk);
      float wsum[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) wsum[k] = 0.f;
#pragma unroll
      for (int ch = 0; ch < 3; ++ch) {
        if (g.drgb[ch] == 0.f) continue;
        const float* shc = pb.sh + static_cast<int64_t>(ch) * pb.sh_k * np + i;
#pragma unroll
        for (int k = 0; k < nk; ++k) {
          wsum[k] = __fmaf_rn(g.drgb[ch], shc[static_cast<int64_t>(k) * np], wsum[k]);
          // dL/dsh_k of this view, rounded once as the separate backward forms it
          sm.shg[ch * nk + k][t] = __fadd_rn(sm.shg[ch * nk + k][t], __fmul_rn(g.drgb[ch], Yk[k]));
        }
      }
      add_view_dir_term<kDeg>(g, wsum);
      const float v[kViewsGeom] = {g.dp[0], g.dp[1], g.dp[2], g.dls[0], g.dls[1], g.dls[2],
                                   g.dq[0], g.dq[1], g.dq[2], g.dq[3], g.dlogit};
#pragma unroll
      for (int j = 0; j < kViewsGeom; ++j) geom[j] = __fadd_rn(geom[j], v[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < kViewsGeom; ++j) sm.geom[j][t] = __fmul_rn(geom[j], a.grad_scale);
#pragma unroll
  for (int c = 0; c < 3 * nk; ++c) sm.shg[c][t] = __fmul_rn(sm.shg[c][t], a.grad_scale);
  __syncthreads();

  // Phase 2: Adam over the CTA's planes; the updated parameters also go to
  // every other rank's buffer.
  auto grad = [&](int pl, const PlaneInfo& info, int col, float4) {
    if (pl < kViewsGeom) return reinterpret_cast<const float4*>(sm.geom[pl])[col];
    return info.k >= 0 ? reinterpret_cast<const float4*>(sm.shg[info.ch * nk + info.k])[col]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  adam_stream<false>(a.f, np, i0, cols, planes, a.base.sh_k, nk, stage, grad, a.copies, a.n_copies);
}

template <int kDeg, bool kMip>
cudaError_t launch_views_mip(const ViewsAdamArgs& a, unsigned grid, cudaStream_t st) {
  const int smem = stage_bytes<false>();
  cudaError_t e = cudaFuncSetAttribute(views_backward_adam_kernel<kDeg, kMip>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_chained(views_backward_adam_kernel<kDeg, kMip>, dim3(grid), dim3(kViewsBlock), smem, st, a);
}

template <int kDeg>
cudaError_t launch_views_deg(const ViewsAdamArgs& a, unsigned grid, cudaStream_t st) {
  return a.base.mip_comp ? launch_views_mip<kDeg, true>(a, grid, st) : launch_views_mip<kDeg, false>(a, grid, st);
}

}  // namespace

cudaError_t launch_views_adam(const ViewsAdamArgs& a, cudaStream_t st) {
  if (a.g_hi <= a.g_lo) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((a.g_hi - a.g_lo + kViewsBlock - 1) / kViewsBlock);
  switch (a.base.active_degree) {
    case 0: return launch_views_deg<0>(a, grid, st);
    case 1: return launch_views_deg<1>(a, grid, st);
    case 2: return launch_views_deg<2>(a, grid, st);
    default: return launch_views_deg<3>(a, grid, st);
  }
}

}  // namespace gs
