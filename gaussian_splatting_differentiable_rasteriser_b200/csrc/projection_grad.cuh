// Per-Gaussian projection backward shared by the kernels that need it: the
// gradient of one visible Gaussian's screen state (from the blend's raw sums)
// with respect to its stored parameters, and optionally the per-Gaussian
// terms of the camera-pose gradient.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), sections "From a pixel's blame to the oval's shape and
// place", "The covariance chain: oval -> 3D ellipsoid -> size & tilt",
// "Where the position gradient comes from" and "Forgiving the camera and the
// light"; "Gaussian splatting training" study notes (bailiping.com), slide "J
// is the 2 x 3 Jacobian of perspective projection".
#pragma once

#include "gs_kernels.cuh"
#include "sh.cuh"

namespace gs {

namespace {

// Gradient of one visible Gaussian with respect to everything but its SH
// coefficients, plus what the SH part needs (masked colour gradient and the
// view direction). The view-direction term of the position is added by
// add_view_dir_term once the SH coefficients have been read.
struct GaussGrad {
  float dp[3], dls[3], dq[4], dlogit;
  float drgb[3];
  float vx, vy, vz, idl;
  float du, dv;  // dL/dmean2d (pixels)
};

// Per-Gaussian terms of the camera-pose gradient (pose update R <- exp([w]x) R,
// t <- t + dt): the camera-frame position gradient dL/dp_c, R p (= p_c - t) and
// the axial vector of Sigma dL/dSigma in the world frame (rotating the camera
// rotates every camera-space covariance).
struct CamTerms {
  float gpc[3];
  float rp[3];
  float ax[3];
};

// kMip: the screen opacity includes the Mip-Splatting compensation factor
// (GS_OPTION_MIP_COMPENSATION); a compile-time switch, so the default
// instantiations carry none of its registers.
template <bool kCam = false, bool kMip = false>
__device__ __forceinline__ void geometry_grad(const PreprocessBwdArgs& a, int64_t i, GaussGrad& out,
                                              CamTerms* ct = nullptr) {
  const int64_t np = a.n_pad;
  const CamArgs& cam = a.cam;
  const float4* sg4 = reinterpret_cast<const float4*>(a.sgrad + i * kGradStride);
  const float4 r0 = sg4[0], r1 = sg4[1], r2 = sg4[2];
  const Screen scr = a.screen[i];
  const float A = conic_A(scr), B = conic_B(scr), C = conic_C(scr), o = screen_opacity(scr);
  const uint8_t clamped = a.clamped[i];

  // Screen-space gradient from the raw sums (w = dL/dalpha * o exp(-e)).
  const float d_u = A * r0.y + B * r0.z;
  const float d_v = B * r0.y + C * r0.z;
  out.du = d_u;
  out.dv = d_v;
  const float dA = -0.5f * r0.w, dB = -r1.x, dC = -0.5f * r1.y;
  const float d_o = o > 0.f ? r0.x / o : 0.f;  // dL/d(screen opacity)
  out.drgb[0] = (clamped & 1) ? 0.f : r1.z;
  out.drgb[1] = (clamped & 2) ? 0.f : r1.w;
  out.drgb[2] = (clamped & 4) ? 0.f : r2.x;
  // screen opacity o = sigmoid(logit) (times comp with the compensation factor)
  const float sig = kMip ? 1.0f / (1.0f + expf(-a.opacity_logits[i])) : o;
  out.dlogit = d_o * o * (1.f - sig);

  // Recompute the forward quantities.
  const float p[3] = {a.means[i], a.means[np + i], a.means[2 * np + i]};
  float pc[3];
#pragma unroll
  for (int r = 0; r < 3; ++r)
    pc[r] = cam.R[3 * r] * p[0] + cam.R[3 * r + 1] * p[1] + cam.R[3 * r + 2] * p[2] + cam.t[r];
  const float X = pc[0], Y = pc[1], Z = pc[2];
  const float qr[4] = {a.quats[i], a.quats[np + i], a.quats[2 * np + i], a.quats[3 * np + i]};
  const float qn = sqrtf(qr[0] * qr[0] + qr[1] * qr[1] + qr[2] * qr[2] + qr[3] * qr[3]);
  const float iqn = 1.0f / qn;
  const float w = qr[0] * iqn, x = qr[1] * iqn, y = qr[2] * iqn, z = qr[3] * iqn;
  const float Rq[9] = {1.f - 2.f * (y * y + z * z), 2.f * (x * y - w * z), 2.f * (x * z + w * y),
                       2.f * (x * y + w * z), 1.f - 2.f * (x * x + z * z), 2.f * (y * z - w * x),
                       2.f * (x * z - w * y), 2.f * (y * z + w * x), 1.f - 2.f * (x * x + y * y)};
  const float s[3] = {expf(a.log_scales[i]), expf(a.log_scales[np + i]),
                      expf(a.log_scales[2 * np + i])};
  float M[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c) M[3 * r + c] = Rq[3 * r + c] * s[c];
  float Sig[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c)
      Sig[3 * r + c] = M[3 * r] * M[3 * c] + M[3 * r + 1] * M[3 * c + 1] + M[3 * r + 2] * M[3 * c + 2];
  const float iz = 1.0f / Z, iz2 = iz * iz;
  const float jx = cam.fx * iz, jy = cam.fy * iz;
  const float jxz = -cam.fx * X * iz2, jyz = -cam.fy * Y * iz2;
  float T[6];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    T[c] = jx * cam.R[c] + jxz * cam.R[6 + c];
    T[3 + c] = jy * cam.R[3 + c] + jyz * cam.R[6 + c];
  }

  // conic -> V': G_V = -K G_K K, G_K = [[dA, dB/2], [dB/2, dC]]
  const float hb = 0.5f * dB;
  const float KG00 = A * dA + B * hb, KG01 = A * hb + B * dC;
  const float KG10 = B * dA + C * hb, KG11 = B * hb + C * dC;
  float GV00 = -(KG00 * A + KG01 * B);
  float GV01 = -(KG00 * B + KG01 * C);
  float GV11 = -(KG10 * B + KG11 * C);
  if (kMip && o > 0.f) {
    // comp = sqrt(det V / det V'), V = T Sigma T^T, V' = V + 0.3 I (the pages'
    // "comp" slot: dL/dcomp = dL/do * sigmoid(logit)); per symmetric entry
    // d comp / dV00 = comp / 2 (V11 / det V - V'11 / det V'), and likewise.
    float V[3] = {0.f, 0.f, 0.f};  // V00, V01, V11
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      const float s0 = Sig[3 * r] * T[0] + Sig[3 * r + 1] * T[1] + Sig[3 * r + 2] * T[2];
      const float s1 = Sig[3 * r] * T[3] + Sig[3 * r + 1] * T[4] + Sig[3 * r + 2] * T[5];
      V[0] += T[r] * s0;
      V[1] += T[r] * s1;
      V[2] += T[3 + r] * s1;
    }
    const float det0 = V[0] * V[2] - V[1] * V[1];
    const float Vd0 = V[0] + kDilationF, Vd2 = V[2] + kDilationF;
    const float det1 = Vd0 * Vd2 - V[1] * V[1];
    if (det0 > 0.f && det1 > 0.f) {
      const float comp = sqrtf(det0 / det1);
      const float k = 0.5f * comp * d_o * sig;
      const float i0 = 1.0f / det0, i1 = 1.0f / det1;
      GV00 += k * (V[2] * i0 - Vd2 * i1);
      GV11 += k * (V[0] * i0 - Vd0 * i1);
      GV01 += k * (V[1] * i1 - V[1] * i0);
    }
  }
  const float GV[4] = {GV00, GV01, GV01, GV11};

  // V' = T Sigma T^T: dSigma = T^T G_V T; dT = 2 G_V T Sigma
  float GVT[6];  // G_V T (2x3)
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    GVT[c] = GV[0] * T[c] + GV[1] * T[3 + c];
    GVT[3 + c] = GV[2] * T[c] + GV[3] * T[3 + c];
  }
  float dSig[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c) dSig[3 * r + c] = T[r] * GVT[c] + T[3 + r] * GVT[3 + c];
  if (kCam) {
    // axial vector of Sigma dL/dSigma (world frame): the camera-rotation term
    float N[9];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
      for (int c = 0; c < 3; ++c)
        N[3 * r + c] = Sig[3 * r] * dSig[c] + Sig[3 * r + 1] * dSig[3 + c] + Sig[3 * r + 2] * dSig[6 + c];
    ct->ax[0] = N[5] - N[7];
    ct->ax[1] = N[6] - N[2];
    ct->ax[2] = N[1] - N[3];
  }
  float dT[6];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c)
      dT[3 * r + c] = 2.f * (GVT[3 * r] * Sig[c] + GVT[3 * r + 1] * Sig[3 + c] + GVT[3 * r + 2] * Sig[6 + c]);
  // T = J W -> dJ = dT W^T; only J00, J02, J11, J12 depend on p_c
  float dJ[6];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c)
      dJ[3 * r + c] = dT[3 * r] * cam.R[3 * c] + dT[3 * r + 1] * cam.R[3 * c + 1] + dT[3 * r + 2] * cam.R[3 * c + 2];
  float dX = dJ[2] * (-cam.fx * iz2);
  float dY = dJ[5] * (-cam.fy * iz2);
  float dZ = dJ[0] * (-cam.fx * iz2) + dJ[2] * (2.f * cam.fx * X * iz2 * iz) +
             dJ[4] * (-cam.fy * iz2) + dJ[5] * (2.f * cam.fy * Y * iz2 * iz);
  // projected mean
  dX += d_u * jx;
  dY += d_v * jy;
  dZ += d_u * jxz + d_v * jyz;
#pragma unroll
  for (int c = 0; c < 3; ++c) out.dp[c] = cam.R[c] * dX + cam.R[3 + c] * dY + cam.R[6 + c] * dZ;
  if (kCam) {
    ct->gpc[0] = dX;
    ct->gpc[1] = dY;
    ct->gpc[2] = dZ;
#pragma unroll
    for (int r = 0; r < 3; ++r) ct->rp[r] = cam.R[3 * r] * p[0] + cam.R[3 * r + 1] * p[1] + cam.R[3 * r + 2] * p[2];
  }

  // Sigma = M M^T -> dM = 2 dSigma M (dSigma symmetric)
  float dM[9];
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c)
      dM[3 * r + c] = 2.f * (dSig[3 * r] * M[c] + dSig[3 * r + 1] * M[3 + c] + dSig[3 * r + 2] * M[6 + c]);
#pragma unroll
  for (int c = 0; c < 3; ++c)
    out.dls[c] = (dM[c] * Rq[c] + dM[3 + c] * Rq[3 + c] + dM[6 + c] * Rq[6 + c]) * s[c];
  float G[9];  // dL/dR = dM diag(s)
#pragma unroll
  for (int r = 0; r < 3; ++r)
#pragma unroll
    for (int c = 0; c < 3; ++c) G[3 * r + c] = dM[3 * r + c] * s[c];
  const float gw = 2.f * (-z * G[1] + y * G[2] + z * G[3] - x * G[5] - y * G[6] + x * G[7]);
  const float gx = 2.f * (y * G[1] + z * G[2] + y * G[3] - 2.f * x * G[4] - w * G[5] + z * G[6] +
                          w * G[7] - 2.f * x * G[8]);
  const float gy = 2.f * (-2.f * y * G[0] + x * G[1] + w * G[2] + x * G[3] + z * G[5] - w * G[6] +
                          z * G[7] - 2.f * y * G[8]);
  const float gz = 2.f * (-2.f * z * G[0] - w * G[1] + x * G[2] + w * G[3] - 2.f * z * G[4] +
                          y * G[5] + x * G[6] + y * G[7]);
  const float qdot = w * gw + x * gx + y * gy + z * gz;
  out.dq[0] = (gw - w * qdot) * iqn;
  out.dq[1] = (gx - x * qdot) * iqn;
  out.dq[2] = (gy - y * qdot) * iqn;
  out.dq[3] = (gz - z * qdot) * iqn;

  // view direction v = normalize(p - campos)
  const float dv[3] = {p[0] - cam.campos[0], p[1] - cam.campos[1], p[2] - cam.campos[2]};
  const float dlen = sqrtf(dv[0] * dv[0] + dv[1] * dv[1] + dv[2] * dv[2]);
  out.idl = 1.0f / dlen;
  out.vx = dv[0] * out.idl;
  out.vy = dv[1] * out.idl;
  out.vz = dv[2] * out.idl;
}

// dp += (dL/dv - v <v, dL/dv>) / |p - campos| with dL/dv = sum_c dL/dc sum_k sh_ck grad Y_k.
template <int kDeg>
__device__ __forceinline__ void add_view_dir_term(GaussGrad& g, const float (&wsum)[16]) {
  float gvx, gvy, gvz;
  sh_grad_dir(kDeg, g.vx, g.vy, g.vz, wsum, gvx, gvy, gvz);
  const float vdot = g.vx * gvx + g.vy * gvy + g.vz * gvz;
  g.dp[0] += (gvx - g.vx * vdot) * g.idl;
  g.dp[1] += (gvy - g.vy * vdot) * g.idl;
  g.dp[2] += (gvz - g.vz * vdot) * g.idl;
}


}  // namespace

}  // namespace gs
