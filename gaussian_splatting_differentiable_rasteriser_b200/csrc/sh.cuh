// Real spherical harmonics up to degree 3 as Cartesian polynomials of the unit
// view direction (x, y, z), with the Condon-Shortley sign pattern the
// taosengine "Gaussian Splats" page prints in its section "Spherical harmonics:
// color that changes with viewing angle" (degree 1 = (-y, z, -x) * 0.4886025).
// Each constant is sqrt2^[m != 0] K_l^|m| |d^|m| P_l / dz^|m||, with
// K_l^m = sqrt((2l+1)/(4 pi) (l-m)!/(l+m)!) and P_l the Legendre polynomial.
// k = 0 is the base colour with basis 1.
#pragma once

namespace gs {

constexpr float kSh1 = 0.48860251190292f;    // sqrt(3 / (4 pi))
constexpr float kSh2a = 1.0925484305920792f;  // sqrt(15 / (4 pi))
constexpr float kSh2b = 0.31539156525252005f; // sqrt(5 / (16 pi))
constexpr float kSh2c = 0.5462742152960396f;  // sqrt(15 / (16 pi))
constexpr float kSh3a = 0.5900435899266436f;  // sqrt(35 / (32 pi))
constexpr float kSh3b = 2.8906114426405547f;  // sqrt(105 / (4 pi))
constexpr float kSh3c = 0.4570457994644658f;  // sqrt(21 / (32 pi))
constexpr float kSh3d = 0.3731763325901154f;  // sqrt(7 / (16 pi))
constexpr float kSh3e = 1.4453057213202773f;  // sqrt(105 / (16 pi))

// Y[k] for k < (degree+1)^2 at unit direction (x, y, z).
__device__ __forceinline__ void sh_basis(int degree, float x, float y, float z, float* Y) {
  Y[0] = 1.0f;
  if (degree < 1) return;
  Y[1] = -kSh1 * y;
  Y[2] = kSh1 * z;
  Y[3] = -kSh1 * x;
  if (degree < 2) return;
  float xx = x * x, yy = y * y, zz = z * z, xy = x * y, yz = y * z, xz = x * z;
  Y[4] = kSh2a * xy;
  Y[5] = -kSh2a * yz;
  Y[6] = kSh2b * (2.0f * zz - xx - yy);
  Y[7] = -kSh2a * xz;
  Y[8] = kSh2c * (xx - yy);
  if (degree < 3) return;
  Y[9] = -kSh3a * y * (3.0f * xx - yy);
  Y[10] = kSh3b * xy * z;
  Y[11] = -kSh3c * y * (4.0f * zz - xx - yy);
  Y[12] = kSh3d * z * (2.0f * zz - 3.0f * xx - 3.0f * yy);
  Y[13] = -kSh3c * x * (4.0f * zz - xx - yy);
  Y[14] = kSh3e * z * (xx - yy);
  Y[15] = -kSh3a * x * (xx - 3.0f * yy);
}

// d/d(x, y, z) of sum_k w[k] Y_k for k = 1 .. (degree+1)^2 - 1 (the polynomial
// forms above, differentiated term by term).
__device__ __forceinline__ void sh_grad_dir(int degree, float x, float y, float z, const float* w,
                                            float& gx, float& gy, float& gz) {
  gx = gy = gz = 0.0f;
  if (degree < 1) return;
  gy += -kSh1 * w[1];
  gz += kSh1 * w[2];
  gx += -kSh1 * w[3];
  if (degree < 2) return;
  float xx = x * x, yy = y * y, zz = z * z, xy = x * y, yz = y * z, xz = x * z;
  gx += kSh2a * y * w[4];
  gy += kSh2a * x * w[4];
  gy += -kSh2a * z * w[5];
  gz += -kSh2a * y * w[5];
  gx += -2.0f * kSh2b * x * w[6];
  gy += -2.0f * kSh2b * y * w[6];
  gz += 4.0f * kSh2b * z * w[6];
  gx += -kSh2a * z * w[7];
  gz += -kSh2a * x * w[7];
  gx += 2.0f * kSh2c * x * w[8];
  gy += -2.0f * kSh2c * y * w[8];
  if (degree < 3) return;
  gx += -6.0f * kSh3a * xy * w[9];
  gy += -3.0f * kSh3a * (xx - yy) * w[9];
  gx += kSh3b * yz * w[10];
  gy += kSh3b * xz * w[10];
  gz += kSh3b * xy * w[10];
  gx += 2.0f * kSh3c * xy * w[11];
  gy += -kSh3c * (4.0f * zz - xx - 3.0f * yy) * w[11];
  gz += -8.0f * kSh3c * yz * w[11];
  gx += -6.0f * kSh3d * xz * w[12];
  gy += -6.0f * kSh3d * yz * w[12];
  gz += kSh3d * (6.0f * zz - 3.0f * xx - 3.0f * yy) * w[12];
  gx += -kSh3c * (4.0f * zz - 3.0f * xx - yy) * w[13];
  gy += 2.0f * kSh3c * xy * w[13];
  gz += -8.0f * kSh3c * xz * w[13];
  gx += 2.0f * kSh3e * xz * w[14];
  gy += -2.0f * kSh3e * yz * w[14];
  gz += kSh3e * (xx - yy) * w[14];
  gx += -3.0f * kSh3a * (xx - yy) * w[15];
  gy += 6.0f * kSh3a * xy * w[15];
}

}  // namespace gs
