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
__device__ __forceinline__ void adam_one(float& p, float& g, float& m, float& v, const AdamScalars& s) {
  m = __fmaf_rn(s.beta1, m, (1.0f - s.beta1) * g);
  v = __fmaf_rn(s.beta2, v, (1.0f - s.beta2) * g * g);
  const float denom = __fmaf_rn(sqrtf(v), s.inv_sqrt_bc2, s.eps);
  p = p - s.step_size * __fdiv_rn(m, denom);
  g = 0.0f;
}

}  // namespace gs
