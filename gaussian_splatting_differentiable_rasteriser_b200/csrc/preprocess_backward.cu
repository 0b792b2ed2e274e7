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
// memory. Phase 2 streams Adam over the CTA's 59 planes x 128 Gaussians: each
// plane segment is 512 contiguous bytes, handled as 32 float4 units, four units
// per thread per round with all 16 loads issued before any store, so many
// loads are in flight per thread (the kernel is bound by HBM, not by math).
constexpr int kFusedBlock = 128;
constexpr int kGeomPlanes = 11;  // means 3, log-scales 3, quats 4, opacity logit 1

constexpr int kMaxPlanes = kGeomPlanes + 3 * 16;

// Where plane pl of the CTA's slice lives: group grp, plane c of that group,
// and for an SH plane its channel ch and coefficient k (k = -1 when the
// coefficient is outside the active bands, so this view adds nothing).
struct PlaneInfo {
  int grp, c, ch, k;
};

// Group, plane within the group, channel and coefficient of plane pl of the
// fused kernel's slice (geometric planes first, then SH channel-major).
__device__ __forceinline__ PlaneInfo plane_info(int pl, int sh_k, int nk) {
  if (pl < 3) return PlaneInfo{0, pl, 0, -1};
  if (pl < 6) return PlaneInfo{1, pl - 3, 0, -1};
  if (pl < 10) return PlaneInfo{2, pl - 6, 0, -1};
  if (pl < 11) return PlaneInfo{3, 0, 0, -1};
  const int sp = pl - kGeomPlanes, ch = sp / sh_k, k = sp % sh_k;
  return PlaneInfo{4, sp, ch, k < nk ? k : -1};
}

#ifndef GS_FUSED_PIPE
#define GS_FUSED_PIPE 1
#endif

// 16-byte asynchronous global -> shared copies (cp.async, L2 only) that each
// thread issues for itself and waits for itself: no CTA barrier is involved.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

struct FusedSmem {
  float geom[kGeomPlanes][kFusedBlock];  // view gradient of the geometric scalars
  float drgb[3][kFusedBlock];            // masked dL/dcolour (0 when invisible)
  float Y[16][kFusedBlock];              // SH basis at the view direction
  PlaneInfo plane[kMaxPlanes];
};

// The pipelined Adam stream. Round r of thread t covers float4 column t % 32 of
// planes t / 32 + 4 R r + 4 s (s < R = kRoundPlanes) of the CTA's slice; its p, (g,) m, v
// are copied with cp.async into the thread's own slots of stage buffer
// r % kStages, kStages rounds ahead of their use, so several planes' loads per
// thread are in flight with no register held for them, and the first rounds
// overlap the projection backward of phase 1. Measured on B200 (Dense, 3M
// Gaussians; Heavy-tail, 6M): 1 plane x 2 stages at 7 CTAs per SM, 0.844 ms
// (1.82 ms); 2 planes x 2 stages at 5 CTAs per SM 0.915 ms; 1 plane x 4
// stages 0.933 ms; 2 planes x 3 stages 1.03 ms; 4 planes x 2 stages (3 CTAs
// per SM) 1.23 ms; the register-staged stream 0.955 ms. Resident CTAs
// matter more than the depth of each one's pipeline.
#ifndef GS_FUSED_ROUND
#define GS_FUSED_ROUND 1
#endif
#ifndef GS_FUSED_STAGES
#define GS_FUSED_STAGES 2
#endif
constexpr int kStages = GS_FUSED_STAGES;  // rounds in flight ahead of the one in use
constexpr int kRoundPlanes = GS_FUSED_ROUND;             // planes per thread per round
constexpr int kRoundStride = (kFusedBlock / 32) * kRoundPlanes;  // planes per round of the CTA
constexpr int kColUnitsF = kFusedBlock / 4;  // float4 columns per plane segment

template <bool kAccum>
constexpr int stage_arrays() { return kAccum ? 4 : 3; }

// slot of (stage buffer, plane s of the round, array) for thread t
template <bool kAccum>
__device__ __forceinline__ float4* stage_slot(float4* stage, int buf, int sidx, int arr) {
  return stage + ((buf * kRoundPlanes + sidx) * stage_arrays<kAccum>() + arr) * kFusedBlock + threadIdx.x;
}

template <bool kAccum>
__device__ __forceinline__ void adam_issue_round(const FusedAdamArgs& f, int64_t np, int64_t i0, int planes,
                                                 int sh_k, int nk, int r, float4* stage) {
  const int t = threadIdx.x, col = t % kColUnitsF;
  const int64_t rem = np - i0;
  const int cols = static_cast<int>((rem < kFusedBlock ? rem : kFusedBlock) / 4);
  if (col < cols) {
#pragma unroll
    for (int sidx = 0; sidx < kRoundPlanes; ++sidx) {
      const int pl = t / kColUnitsF + kRoundStride * r + 4 * sidx;
      if (pl >= planes) continue;
      const PlaneInfo info = plane_info(pl, sh_k, nk);
      const int64_t off = static_cast<int64_t>(info.c) * np + i0 + 4 * col;
      const int buf = r % kStages;
      cp_async16(stage_slot<kAccum>(stage, buf, sidx, 0), f.p[info.grp] + off);
      if (kAccum) cp_async16(stage_slot<kAccum>(stage, buf, sidx, 3), f.g[info.grp] + off);
      cp_async16(stage_slot<kAccum>(stage, buf, sidx, 1), f.m[info.grp] + off);
      cp_async16(stage_slot<kAccum>(stage, buf, sidx, 2), f.v[info.grp] + off);
    }
  }
  cp_async_commit();  // one group per round, empty or not
}

template <bool kAccum>
__device__ __forceinline__ void adam_stream_pipelined(const FusedSmem& sm, const FusedAdamArgs& f, int64_t np,
                                                      int64_t i0, int planes, float4* stage) {
  const int t = threadIdx.x, col = t % kColUnitsF;
  const int64_t rem = np - i0;
  const int cols = static_cast<int>((rem < kFusedBlock ? rem : kFusedBlock) / 4);
  const bool col_ok = col < cols;
  const int rounds = (planes + kRoundStride - 1) / kRoundStride;
  for (int r = 0; r < rounds; ++r) {
    cp_async_wait<kStages - 1>();  // this thread's copies of round r have landed (later rounds may be pending)
    const int buf = r % kStages;
    float4 P[kRoundPlanes], G[kRoundPlanes], M[kRoundPlanes], V[kRoundPlanes];
    PlaneInfo info[kRoundPlanes];
#pragma unroll
    for (int sidx = 0; sidx < kRoundPlanes; ++sidx) {
      const int pl = t / kColUnitsF + kRoundStride * r + 4 * sidx;
      info[sidx] = sm.plane[pl < planes ? pl : 0];
      G[sidx] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col_ok && pl < planes) {
        P[sidx] = *stage_slot<kAccum>(stage, buf, sidx, 0);
        M[sidx] = *stage_slot<kAccum>(stage, buf, sidx, 1);
        V[sidx] = *stage_slot<kAccum>(stage, buf, sidx, 2);
        if (kAccum) G[sidx] = *stage_slot<kAccum>(stage, buf, sidx, 3);
      }
    }
#pragma unroll
    for (int sidx = 0; sidx < kRoundPlanes; ++sidx) {
      const int pl = t / kColUnitsF + kRoundStride * r + 4 * sidx;
      if (!col_ok || pl >= planes) continue;
      float* p4 = &P[sidx].x;
      float* g4 = &G[sidx].x;
      float* m4 = &M[sidx].x;
      float* v4 = &V[sidx].x;
      const AdamScalars sc = f.s[info[sidx].grp];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * col + e;
        if (pl < kGeomPlanes) {
          g4[e] += sm.geom[pl][j];
        } else if (info[sidx].k >= 0) {
          const float dc = sm.drgb[info[sidx].ch][j];
          if (dc != 0.f) g4[e] = __fmaf_rn(dc, sm.Y[info[sidx].k][j], g4[e]);
        }
        adam_one(p4[e], g4[e], m4[e], v4[e], sc);
      }
      const int64_t off = static_cast<int64_t>(info[sidx].c) * np + i0 + 4 * col;
      *reinterpret_cast<float4*>(f.p[info[sidx].grp] + off) = P[sidx];
      if (kAccum) *reinterpret_cast<float4*>(f.g[info[sidx].grp] + off) = G[sidx];
      *reinterpret_cast<float4*>(f.m[info[sidx].grp] + off) = M[sidx];
      *reinterpret_cast<float4*>(f.v[info[sidx].grp] + off) = V[sidx];
    }
    // refill this stage buffer with round r + kStages (its old values are in
    // registers and already consumed by the stores above)
    if (r + kStages < rounds) {
      if (col_ok) {
#pragma unroll
        for (int sidx = 0; sidx < kRoundPlanes; ++sidx) {
          const int pl = t / kColUnitsF + kRoundStride * (r + kStages) + 4 * sidx;
          if (pl >= planes) continue;
          const PlaneInfo in2 = sm.plane[pl];
          const int64_t off = static_cast<int64_t>(in2.c) * np + i0 + 4 * col;
          cp_async16(stage_slot<kAccum>(stage, buf, sidx, 0), f.p[in2.grp] + off);
          if (kAccum) cp_async16(stage_slot<kAccum>(stage, buf, sidx, 3), f.g[in2.grp] + off);
          cp_async16(stage_slot<kAccum>(stage, buf, sidx, 1), f.m[in2.grp] + off);
          cp_async16(stage_slot<kAccum>(stage, buf, sidx, 2), f.v[in2.grp] + off);
        }
      }
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
}

// kAccum: the caller's gradient buffer holds an accumulated gradient, which is
// added and then zeroed; without it the update uses this view's gradient alone
// and no gradient buffer is read or written (24 instead of 32 bytes per scalar).
template <int kDeg, bool kAccum, bool kStats, bool kMip>
__global__ void __launch_bounds__(kFusedBlock) preprocess_backward_adam_kernel(PreprocessBwdArgs a,
                                                                              FusedAdamArgs f) {
  __shared__ __align__(16) FusedSmem sm;
  const int t = threadIdx.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kFusedBlock;
  const int64_t np = a.n_pad;
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
#if GS_FUSED_PIPE
  // The first two rounds of the Adam stream are in flight while phase 1 runs.
  extern __shared__ __align__(16) float4 stage[];
  {
    const int planes = kGeomPlanes + 3 * a.sh_k;
#pragma unroll
    for (int r = 0; r < kStages; ++r) adam_issue_round<kAccum>(f, np, i0, planes, a.sh_k, nk, r, stage);
  }
#endif

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
  if (t < kGeomPlanes + 3 * a.sh_k) sm.plane[t] = plane_info(t, a.sh_k, nk);
  __syncthreads();
#if GS_FUSED_PIPE
  adam_stream_pipelined<kAccum>(sm, f, np, i0, kGeomPlanes + 3 * a.sh_k, stage);
  return;
#endif

  // Phase 2: Adam over planes x float4 columns of this CTA's Gaussians. Thread
  // t takes float4 column t % 32 of planes t / 32, t / 32 + 4, ...; four planes
  // per round with all their loads issued before any store. Plane bookkeeping
  // comes from the table built in phase 1 (one broadcast load per plane).
  const int64_t rem = np - i0;
  const int cols = static_cast<int>((rem < kFusedBlock ? rem : kFusedBlock) / 4);  // n_pad % 4 == 0
  const int planes = kGeomPlanes + 3 * a.sh_k;
  constexpr int kColUnits = kFusedBlock / 4;            // float4 columns per plane
  constexpr int kPlaneStep = kFusedBlock / kColUnits;   // planes per sweep of the CTA
  const int col = t % kColUnits;
  const bool col_ok = col < cols;
  for (int pl0 = t / kColUnits; pl0 < planes; pl0 += 4 * kPlaneStep) {
    float4 P[4], G[4], M[4], V[4];
    PlaneInfo info[4];
    int64_t off[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int pl = pl0 + r * kPlaneStep;
      const bool ok = col_ok && pl < planes;
      info[r] = sm.plane[pl < planes ? pl : 0];
      off[r] = static_cast<int64_t>(info[r].c) * np + i0 + 4 * col;
      G[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok) {
        P[r] = *reinterpret_cast<const float4*>(f.p[info[r].grp] + off[r]);
        if (kAccum) G[r] = *reinterpret_cast<const float4*>(f.g[info[r].grp] + off[r]);
        M[r] = *reinterpret_cast<const float4*>(f.m[info[r].grp] + off[r]);
        V[r] = *reinterpret_cast<const float4*>(f.v[info[r].grp] + off[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int pl = pl0 + r * kPlaneStep;
      if (!col_ok || pl >= planes) continue;
      float* p4 = &P[r].x;
      float* g4 = &G[r].x;
      float* m4 = &M[r].x;
      float* v4 = &V[r].x;
      const AdamScalars sc = f.s[info[r].grp];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * col + e;
        if (pl < kGeomPlanes) {
          g4[e] += sm.geom[pl][j];
        } else if (info[r].k >= 0) {
          const float dc = sm.drgb[info[r].ch][j];
          if (dc != 0.f) g4[e] = __fmaf_rn(dc, sm.Y[info[r].k][j], g4[e]);
        }
        adam_one(p4[e], g4[e], m4[e], v4[e], sc);
      }
      *reinterpret_cast<float4*>(f.p[info[r].grp] + off[r]) = P[r];
      if (kAccum) *reinterpret_cast<float4*>(f.g[info[r].grp] + off[r]) = G[r];
      *reinterpret_cast<float4*>(f.m[info[r].grp] + off[r]) = M[r];
      *reinterpret_cast<float4*>(f.v[info[r].grp] + off[r]) = V[r];
    }
  }
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
  // the pipelined stream's stage buffers: kStages rounds x kRoundPlanes planes x (3 or 4) arrays x 128 float4
  const int smem = GS_FUSED_PIPE ? kStages * kRoundPlanes * stage_arrays<kAccum>() * kFusedBlock * 16 : 0;
  cudaError_t e = cudaFuncSetAttribute(preprocess_backward_adam_kernel<kDeg, kAccum, kStats, kMip>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  preprocess_backward_adam_kernel<kDeg, kAccum, kStats, kMip><<<grid, kFusedBlock, smem, st>>>(a, f);
  return cudaGetLastError();
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
