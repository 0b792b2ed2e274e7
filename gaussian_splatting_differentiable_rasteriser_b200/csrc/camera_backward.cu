// Camera-pose gradient of one view: dL/dw and dL/dt for the pose update
// R <- exp([w]x) R, t <- t + dt.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), section "Forgiving the camera and the light": the render
// depends on the camera, so backprop gives it a gradient. That section's code
// sums, per Gaussian, the rotation blame cross(p_c - t, dL/dp_c) and the
// translation blame dL/dp_c. The gradient here is the exact one of that
// parametrisation, with two further paths the section leaves out:
//   * rotating the camera rotates every camera-space covariance
//     Sigma_c = W Sigma W^T: dL/dw += 2 W axial(Sigma dL/dSigma);
//   * the camera centre campos = -R^T t moves (the colour's view direction):
//     with c = sum_i dL/dcampos_i = -sum_i (view-direction part of dL/dp_i),
//     dL/dw += t x (R c) and dL/dt -= R c.
//
// B200 design: one pass over the Gaussians on a fixed grid of 148 x 3 CTAs,
// one wave at 3 CTAs per SM (80 registers; the per-Gaussian chain of dependent
// loads is latency-bound, so resident warps count), grid-stride, reusing the
// projection backward's per-Gaussian algebra; each
// thread sums its Gaussians' nine terms in float64, each CTA reduces them in a
// fixed order, and the last CTA to finish adds the CTAs' partial sums in a
// fixed order and forms the six outputs, so the result is deterministic for
// a given screen gradient. It reads about 150 B per visible Gaussian (the
// parameters, the screen record, the raw sums and the SH coefficients of
// colours that received a gradient) and writes 48 B.
#include "gs_kernels.cuh"
#include "projection_grad.cuh"
#include "sh.cuh"

namespace gs {

namespace {

constexpr int kCamThreads = 256;

template <int kDeg, bool kMip>
__global__ void __launch_bounds__(kCamThreads, 3) camera_backward_kernel(PreprocessBwdArgs a, CameraGradArgs cg) {
  __shared__ double s_red[9][kCamThreads / 32];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t np = a.n_pad;
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
  double acc[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};  // rotation 3, translation 3, campos 3
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kCamThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kCamThreads + tid; i < a.n; i += stride) {
    if (a.touched[i] == 0) continue;
    GaussGrad g;
    CamTerms ct;
    geometry_grad<true, kMip>(a, i, g, &ct);
    // view-direction part of dL/dp: (dL/dv - v <v, dL/dv>) / |p - campos|
    float wsum[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) wsum[k] = 0.f;
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) {
      if (g.drgb[ch] == 0.f) continue;
      const float* shc = a.sh + static_cast<int64_t>(ch) * a.sh_k * np + i;
#pragma unroll
      for (int k = 0; k < nk; ++k) wsum[k] = __fmaf_rn(g.drgb[ch], shc[static_cast<int64_t>(k) * np], wsum[k]);
    }
    float gvx, gvy, gvz;
    sh_grad_dir(kDeg, g.vx, g.vy, g.vz, wsum, gvx, gvy, gvz);
    const float vdot = g.vx * gvx + g.vy * gvy + g.vz * gvz;
    const float vd[3] = {(gvx - g.vx * vdot) * g.idl, (gvy - g.vy * vdot) * g.idl, (gvz - g.vz * vdot) * g.idl};
    // rotation: (R p) x dL/dp_c + 2 R axial(Sigma dL/dSigma)
    const float* R = a.cam.R;
    const float tq[3] = {ct.rp[1] * ct.gpc[2] - ct.rp[2] * ct.gpc[1], ct.rp[2] * ct.gpc[0] - ct.rp[0] * ct.gpc[2],
                         ct.rp[0] * ct.gpc[1] - ct.rp[1] * ct.gpc[0]};
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      const float rot = R[3 * r] * ct.ax[0] + R[3 * r + 1] * ct.ax[1] + R[3 * r + 2] * ct.ax[2];
      acc[r] += static_cast<double>(tq[r]) + 2.0 * static_cast<double>(rot);
      acc[3 + r] += ct.gpc[r];
      acc[6 + r] -= vd[r];  // dL/dcampos
    }
  }
  // CTA sums in a fixed order
#pragma unroll
  for (int k = 0; k < 9; ++k) {
    double v = acc[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_red[k][warp] = v;
  }
  __syncthreads();
  if (tid < 9) {
    double t = 0.0;
    for (int w = 0; w < kCamThreads / 32; ++w) t += s_red[tid][w];
    cg.partials[9 * blockIdx.x + tid] = t;
    __threadfence();
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(cg.counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (tid == 0) {
    double tot[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
    for (unsigned b = 0; b < gridDim.x; ++b)
      for (int k = 0; k < 9; ++k) tot[k] += __ldcg(cg.partials + 9 * b + k);
    const float* R = a.cam.R;
    const float* t = a.cam.t;
    double Rc[3];
    for (int r = 0; r < 3; ++r)
      Rc[r] = static_cast<double>(R[3 * r]) * tot[6] + static_cast<double>(R[3 * r + 1]) * tot[7] +
              static_cast<double>(R[3 * r + 2]) * tot[8];
    const double t0 = t[0], t1 = t[1], t2 = t[2];
    cg.out[0] = tot[0] + (t1 * Rc[2] - t2 * Rc[1]);
    cg.out[1] = tot[1] + (t2 * Rc[0] - t0 * Rc[2]);
    cg.out[2] = tot[2] + (t0 * Rc[1] - t1 * Rc[0]);
    cg.out[3] = tot[3] - Rc[0];
    cg.out[4] = tot[4] - Rc[1];
    cg.out[5] = tot[5] - Rc[2];
    *cg.counter = 0u;  // ready for the next view
  }
}

template <int kDeg>
cudaError_t launch_cam_deg(const PreprocessBwdArgs& a, const CameraGradArgs& g, cudaStream_t st) {
  const int64_t want = (a.n + kCamThreads - 1) / kCamThreads;
  const unsigned grid = static_cast<unsigned>(want < kCamBlocks ? (want > 0 ? want : 1) : kCamBlocks);
  if (a.mip_comp)
    camera_backward_kernel<kDeg, true><<<grid, kCamThreads, 0, st>>>(a, g);
  else
    camera_backward_kernel<kDeg, false><<<grid, kCamThreads, 0, st>>>(a, g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_camera_backward(const PreprocessBwdArgs& a, const CameraGradArgs& g, cudaStream_t st) {
  switch (a.active_degree) {
    case 0: return launch_cam_deg<0>(a, g, st);
    case 1: return launch_cam_deg<1>(a, g, st);
    case 2: return launch_cam_deg<2>(a, g, st);
    default: return launch_cam_deg<3>(a, g, st);
  }
}

}  // namespace gs
