// The per-scalar Adam update shared by the standalone Adam kernel and the
// fused projection-backward + Adam kernel, so both produce identical bits.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), Adam paragraph after "Proving the blame is right".
#pragma once

namespace gs {

struct AdamScalars {
  float step_size;     // lr / (1 - b1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
  float beta1, beta2, eps;
};

// m = b1 m + (1 - b1) g; v = b2 v + (1 - b2) g^2;
// p -= lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps); g = 0.
// Every rounding step is an explicit intrinsic, so each kernel that inlines
// this produces the same bits whatever the compiler contracts around it. The
// square root and the division use the hardware approximations (sqrt.approx,
// __fdividef: a few ulp): the update p -= step m / denom then carries a
// relative error near 1e-7 of a step of about lr, where IEEE-rounded sqrt and
// division would cost tens of instructions per scalar - most of the issue
// slots of the streaming Adam passes.
__device__ __forceinline__ float sqrt_approx(float x) {
  float y;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void adam_one(float& p, float& g, float& m, float& v, const AdamScalars& s) {
  m = __fmaf_rn(s.beta1, m, __fmul_rn(1.0f - s.beta1, g));
  v = __fmaf_rn(s.beta2, v, __fmul_rn(__fmul_rn(1.0f - s.beta2, g), g));
  const float denom = __fmaf_rn(sqrt_approx(v), s.inv_sqrt_bc2, s.eps);
  p = __fmaf_rn(-s.step_size, __fdividef(m, denom), p);
  g = 0.0f;
}

}  // namespace gs
