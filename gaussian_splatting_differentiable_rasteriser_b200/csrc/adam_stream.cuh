// The Adam pass over one CTA's slice of the planar parameter buffers, shared by
// the fused projection backward + Adam kernel and the data-parallel update from
// the views' screen sums.
//
// A CTA owns 128 consecutive Gaussians; its slice is 11 geometric planes
// (means 3, log-scales 3, quats 4, opacity logit 1) and 3 x sh_k SH planes of
// 128 floats each. Round r of thread t covers float4 column t % 32 of planes
// t / 32 + 4 R r + 4 s (s < R = kRoundPlanes). Its p, (g,) m, v are copied
// with cp.async into the thread's own slots of stage buffer r % kStages,
// kStages rounds ahead of their use, so several planes' loads per thread are
// in flight with no register held for them, and the first rounds (issued
// before the kernel's per-Gaussian phase) overlap that phase. Each thread
// waits only for its own copies: no CTA barrier is involved.
//
// Measured on B200 (Dense, 3M Gaussians; Heavy-tail, 6M), for the fused
// kernel: 1 plane x 2 stages at 7 CTAs per SM, 0.844 ms (1.82 ms); 2 planes x
// 2 stages at 5 CTAs per SM 0.915 ms; 1 plane x 4 stages 0.933 ms; 2 planes x
// 3 stages 1.03 ms; 4 planes x 2 stages (3 CTAs per SM) 1.23 ms; a
// register-staged stream with 16 loads in flight per thread 0.955 ms.
// Resident CTAs matter more than the depth of each one's pipeline. With
// Adam's hardware division and each round's plane info computed in registers
// instead of read from a shared-memory table: 0.749 ms (1.45 ms).
#pragma once

#include "adam_math.cuh"
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kStreamBlock = 128;   // Gaussians (and threads) per CTA
constexpr int kStreamGeom = 11;     // geometric planes

#ifndef GS_FUSED_ROUND
#define GS_FUSED_ROUND 1
#endif
#ifndef GS_FUSED_STAGES
#define GS_FUSED_STAGES 2
#endif
constexpr int kStages = GS_FUSED_STAGES;                           // rounds in flight ahead of the one in use
constexpr int kRoundPlanes = GS_FUSED_ROUND;                       // planes per thread per round
constexpr int kRoundStride = (kStreamBlock / 32) * kRoundPlanes;   // planes per round of the CTA
constexpr int kColUnits = kStreamBlock / 4;                        // float4 columns per plane segment

// Where plane pl of the slice lives: group grp, plane c of that group, and for
// an SH plane its channel ch and coefficient k (k = -1 outside the active bands).
struct PlaneInfo {
  int grp, c, ch, k;
};

__device__ __forceinline__ PlaneInfo plane_info(int pl, int sh_k, int nk) {
  if (pl < 3) return PlaneInfo{0, pl, 0, -1};
  if (pl < 6) return PlaneInfo{1, pl - 3, 0, -1};
  if (pl < 10) return PlaneInfo{2, pl - 6, 0, -1};
  if (pl < 11) return PlaneInfo{3, 0, 0, -1};
  const int sp = pl - kStreamGeom;
  const int ch = (sp >= sh_k) + (sp >= 2 * sh_k);  // sp < 3 sh_k
  const int k = sp - ch * sh_k;
  return PlaneInfo{4, sp, ch, k < nk ? k : -1};
}

// 16-byte asynchronous global -> shared copies (cp.async, L2 only) that each
// thread issues for itself and waits for itself.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <bool kAccum>
constexpr int stage_arrays() { return kAccum ? 4 : 3; }

// Bytes of dynamic shared memory the stage buffers take.
template <bool kAccum>
constexpr int stage_bytes() { return kStages * kRoundPlanes * stage_arrays<kAccum>() * kStreamBlock * 16; }

// Slot of (stage buffer, plane s of the round, array) for this thread.
template <bool kAccum>
__device__ __forceinline__ float4* stage_slot(float4* stage, int buf, int sidx, int arr) {
  return stage + ((buf * kRoundPlanes + sidx) * stage_arrays<kAccum>() + arr) * kStreamBlock + threadIdx.x;
}

// Float4 columns of the slice that start at i0 and end before `end` (a multiple of 4).
__device__ __forceinline__ int stream_cols(int64_t i0, int64_t end) {
  const int64_t rem = end - i0;
  return static_cast<int>((rem < kStreamBlock ? rem : kStreamBlock) / 4);
}

template <bool kAccum>
__device__ __forceinline__ void adam_issue_round(const FusedAdamArgs& f, int64_t np, int64_t i0, int cols,
                                                 int planes, int sh_k, int nk, int r, float4* stage) {
  const int t = threadIdx.x, col = t % kColUnits;
  if (col < cols) {
#pragma unroll
    for (int sidx = 0; sidx < kRoundPlanes; ++sidx) {
      const int pl = t / kColUnits + kRoundStride * r + 4 * sidx;
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

// The first kStages rounds, issued before the kernel's per-Gaussian phase.
template <bool kAccum>
__device__ __forceinline__ void adam_stream_prologue(const FusedAdamArgs& f, int64_t np, int64_t i0, int cols,
                                                     int planes, int sh_k, int nk, float4* stage) {
#pragma unroll
  for (int r = 0; r < kStages; ++r) adam_issue_round<kAccum>(f, np, i0, cols, planes, sh_k, nk, r, stage);
}

// The stream proper. grad(pl, info, col, g) returns the gradients of plane pl
// at the slice's Gaussians 4 col .. 4 col + 3, given g (the accumulated
// gradients, 0 without them);
// the updated parameters also go to each of the n_copies parameter buffers.
// Each round's plane_info is computed from the plane index (a few compares)
// rather than read from a table in shared memory: the stores' addresses then
// do not wait on a shared-memory load (Dense fused pass 0.822 -> 0.749 ms).
template <bool kAccum, class Grad>
__device__ __forceinline__ void adam_stream(const FusedAdamArgs& f, int64_t np,
                                            int64_t i0, int cols, int planes, int sh_k, int nk, float4* stage,
                                            const Grad& grad, float* const (*copies)[5] = nullptr,
                                            int n_copies = 0) {
  const int t = threadIdx.x, col = t % kColUnits;
  const bool col_ok = col < cols;
  const int rounds = (planes + kRoundStride - 1) / kRoundStride;
  for (int r = 0; r < rounds; ++r) {
    cp_async_wait<kStages - 1>();  // this thread's copies of round r have landed (later rounds may be pending)
    const int buf = r % kStages;
    float4 P[kRoundPlanes], G[kRoundPlanes], M[kRoundPlanes], V[kRoundPlanes];
    PlaneInfo info[kRoundPlanes];
#pragma unroll
    for (int sidx = 0; sidx < kRoundPlanes; ++sidx) {
      const int pl = t / kColUnits + kRoundStride * r + 4 * sidx;
      info[sidx] = plane_info(pl < planes ? pl : 0, sh_k, nk);
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
      const int pl = t / kColUnits + kRoundStride * r + 4 * sidx;
      if (!col_ok || pl >= planes) continue;
      float* p4 = &P[sidx].x;
      float* g4 = &G[sidx].x;
      float* m4 = &M[sidx].x;
      float* v4 = &V[sidx].x;
      const AdamScalars sc = f.s[info[sidx].grp];
      G[sidx] = grad(pl, info[sidx], col, G[sidx]);
#pragma unroll
      for (int e = 0; e < 4; ++e) adam_one(p4[e], g4[e], m4[e], v4[e], sc);
      const int64_t off = static_cast<int64_t>(info[sidx].c) * np + i0 + 4 * col;
      *reinterpret_cast<float4*>(f.p[info[sidx].grp] + off) = P[sidx];
      if (kAccum) *reinterpret_cast<float4*>(f.g[info[sidx].grp] + off) = G[sidx];
      *reinterpret_cast<float4*>(f.m[info[sidx].grp] + off) = M[sidx];
      *reinterpret_cast<float4*>(f.v[info[sidx].grp] + off) = V[sidx];
      for (int d = 0; d < n_copies; ++d) *reinterpret_cast<float4*>(copies[d][info[sidx].grp] + off) = P[sidx];
    }
    // refill this stage buffer with round r + kStages (its old values are in
    // registers and already consumed by the stores above)
    if (r + kStages < rounds) adam_issue_round<kAccum>(f, np, i0, cols, planes, sh_k, nk, r + kStages, stage);
    else cp_async_commit();
  }
  cp_async_wait<0>();
}

}  // namespace

}  // namespace gs
