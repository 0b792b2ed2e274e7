// Fused photometric loss (1 - lambda) L1 + lambda (1 - SSIM) and its pixel
// gradient in one kernel.
//
// Method: "Gaussian splatting training" study notes (bailiping.com), slides on
// the loss (lambda = 0.2, no 1/2 on D-SSIM), L1 (mean over 3HW, zero
// subgradient at zero residual) and SSIM (11x11 Gaussian window of sigma 1.5,
// C1 = 0.01^2, C2 = 0.03^2, zero padding, mean over pixels and channels).
// The SSIM gradient couples neighbours through the window moments:
//   dSSIM/dx_p = 1/(3HW) sum_q w(q - p) [dS_q/dmu_x + 2 x_p dS_q/dE[x^2] + y_p dS_q/dE[xy]].
//
// B200 design: one CTA per 32x32 output tile and channel does everything in
// shared memory with halo recompute - no intermediate maps in HBM, so the
// kernel reads the two images once and writes the gradient once (36 B per
// pixel over the three channels). Every filter pass is register-tiled: a
// thread produces 4 (or 4 x 2) consecutive outputs from a window it loads once
// with vector loads, so shared memory serves several times fewer loads than
// one per tap; the squared and cross products are formed once per window
// element. The adjoint buffer reuses the horizontal-moment buffer once that is
// dead (about 90 KB per CTA). Steps: load the 52x52 input region (zero outside
// the image), separable 11-tap horizontal then vertical filtering of the 5
// moments over the 42x42 region of SSIM-map positions the tile's gradient
// depends on, the map and its three partial derivatives there (zero outside
// the image), then the separable adjoint filter back onto the 32x32 tile.
// Block partial sums of |x - y| and of the map go to a small array that the
// last CTA to finish reduces in a fixed order in float64, so the loss is
// deterministic.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kOut = 32;                 // output tile side
constexpr int kR = 5;                    // window radius
constexpr int kQ = kOut + 2 * kR;        // 42: SSIM-map positions needed
constexpr int kIn = kOut + 4 * kR;       // 52: input pixels needed
constexpr int kQs = 44;                  // padded row stride of the 42-wide maps (16 B rows)
constexpr int kLossThreads = 256;
static_assert(kQs >= kQ && kQs % 4 == 0, "map rows must hold the 42 columns and stay 16-byte aligned");

struct LossSmem {
  float x[kIn * kIn];
  float y[kIn * kIn];
  union {
    float h[5][kIn * kQs];   // horizontal moments: input rows x map columns
    float a[3][kQ * kOut];   // (after the vertical pass) horizontally filtered partials
  };
  float d[3][kQ * kQs];  // map partials dS/dmu_x, dS/dE[x^2], dS/dE[xy]
  double red[2][kLossThreads / 32];
  int last;
};

__device__ __forceinline__ void load4(const float* p, float* v) {
  const float4 t = *reinterpret_cast<const float4*>(p);
  v[0] = t.x;
  v[1] = t.y;
  v[2] = t.z;
  v[3] = t.w;
}

__global__ void __launch_bounds__(kLossThreads) loss_kernel(LossArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  LossSmem& s = *reinterpret_cast<LossSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int x0 = blockIdx.x * kOut, y0 = blockIdx.y * kOut;
  const int H = a.height, W = a.width;
  const int64_t HW = static_cast<int64_t>(H) * W;
  const float inv = static_cast<float>(1.0 / (3.0 * static_cast<double>(HW)));
  const float C1 = 0.01f * 0.01f, C2 = 0.03f * 0.03f;
  float l1_acc = 0.0f, ssim_acc = 0.0f;
  float w[2 * kR + 1];
#pragma unroll
  for (int t = 0; t <= 2 * kR; ++t) w[t] = a.window[t];

  const int ch = blockIdx.z;
  const float* X = a.x + ch * HW;
  const float* Yc = a.y + ch * HW;
  // 1. input region [y0 - 10, y0 + 42) x [x0 - 10, x0 + 42), zero padded
  for (int k = tid; k < kIn * kIn; k += kLossThreads) {
    const int r = k / kIn, c = k % kIn;
    const int gy = y0 - 2 * kR + r, gx = x0 - 2 * kR + c;
    const bool in = gy >= 0 && gy < H && gx >= 0 && gx < W;
    const int64_t g = static_cast<int64_t>(gy) * W + gx;
    s.x[k] = in ? __ldg(X + g) : 0.0f;
    s.y[k] = in ? __ldg(Yc + g) : 0.0f;
  }
  __syncthreads();
  // 2. horizontal moments, 4 map columns per item from a 16-wide window in
  //    registers; map column j <-> image x0 - 5 + j
  for (int it = tid; it < kIn * 11; it += kLossThreads) {
    const int r = it / 11, j0 = 4 * (it % 11);
    float xv[16], yv[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = j0 + 4 * q;
      if (c < kIn) {
        load4(s.x + r * kIn + c, xv + 4 * q);
        load4(s.y + r * kIn + c, yv + 4 * q);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) xv[4 * q + e] = yv[4 * q + e] = 0.f;
      }
    }
    float pxx[14], pyy[14], pxy[14];  // products once per window element
#pragma unroll
    for (int e = 0; e < 14; ++e) {
      pxx[e] = xv[e] * xv[e];
      pyy[e] = yv[e] * yv[e];
      pxy[e] = xv[e] * yv[e];
    }
    float m[5][4];
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      float mx = 0.f, my = 0.f, mxx = 0.f, myy = 0.f, mxy = 0.f;
#pragma unroll
      for (int t = 0; t <= 2 * kR; ++t) {
        mx = __fmaf_rn(w[t], xv[o + t], mx);
        my = __fmaf_rn(w[t], yv[o + t], my);
        mxx = __fmaf_rn(w[t], pxx[o + t], mxx);
        myy = __fmaf_rn(w[t], pyy[o + t], myy);
        mxy = __fmaf_rn(w[t], pxy[o + t], mxy);
      }
      m[0][o] = mx;
      m[1][o] = my;
      m[2][o] = mxx;
      m[3][o] = myy;
      m[4][o] = mxy;
    }
#pragma unroll
    for (int c = 0; c < 5; ++c)
      *reinterpret_cast<float4*>(s.h[c] + r * kQs + j0) = make_float4(m[c][0], m[c][1], m[c][2], m[c][3]);
  }
  __syncthreads();
  // 3. vertical pass (2 map columns x 4 map rows per item), SSIM map and its
  //    partial derivatives at the 42x42 positions
  for (int it = tid; it < 21 * 11; it += kLossThreads) {
    const int qj = 2 * (it % 21), qi0 = 4 * (it / 21);
    float acc[5][4][2];
#pragma unroll
    for (int c = 0; c < 5; ++c)
#pragma unroll
      for (int o = 0; o < 4; ++o) acc[c][o][0] = acc[c][o][1] = 0.f;
#pragma unroll
    for (int rr = 0; rr < 14; ++rr) {
      const int row = qi0 + rr;
      if (row >= kIn) break;
#pragma unroll
      for (int c = 0; c < 5; ++c) {
        const float2 hv = *reinterpret_cast<const float2*>(s.h[c] + row * kQs + qj);
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const int t = rr - o;
          if (t >= 0 && t <= 2 * kR) {
            acc[c][o][0] = __fmaf_rn(w[t], hv.x, acc[c][o][0]);
            acc[c][o][1] = __fmaf_rn(w[t], hv.y, acc[c][o][1]);
          }
        }
      }
    }
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const int qi = qi0 + o;
      if (qi >= kQ) break;
      float dm2[2], dxx2[2], dxy2[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int qje = qj + e;
        const int gy = y0 - kR + qi, gx = x0 - kR + qje;
        float dm = 0.f, dxx = 0.f, dxy = 0.f;
        if (gy >= 0 && gy < H && gx >= 0 && gx < W) {
          const float mux = acc[0][o][e], muy = acc[1][o][e];
          const float sxx = acc[2][o][e] - mux * mux, syy = acc[3][o][e] - muy * muy;
          const float sxy = acc[4][o][e] - mux * muy;
          const float A1 = 2.f * mux * muy + C1, A2 = 2.f * sxy + C2;
          const float B1 = mux * mux + muy * muy + C1, B2 = sxx + syy + C2;
          const float iB1 = 1.0f / B1, iB2 = 1.0f / B2;
          const float iB = iB1 * iB2;
          const float S = A1 * A2 * iB;
          // partials with mu_y, E[y^2] fixed: sxx = E[x^2] - mux^2, sxy = E[xy] - mux muy
          dm = 2.f * muy * (A2 - A1) * iB - 2.f * mux * S * (iB1 - iB2);
          dxx = -S * iB2;
          dxy = 2.f * A1 * iB;
          if (qi >= kR && qi < kR + kOut && qje >= kR && qje < kR + kOut) ssim_acc += S;
        }
        dm2[e] = dm;
        dxx2[e] = dxx;
        dxy2[e] = dxy;
      }
      *reinterpret_cast<float2*>(s.d[0] + qi * kQs + qj) = make_float2(dm2[0], dm2[1]);
      *reinterpret_cast<float2*>(s.d[1] + qi * kQs + qj) = make_float2(dxx2[0], dxx2[1]);
      *reinterpret_cast<float2*>(s.d[2] + qi * kQs + qj) = make_float2(dxy2[0], dxy2[1]);
    }
  }
  __syncthreads();
  // 4. horizontal adjoint onto the output columns (the window is symmetric):
  //    4 output columns per item from a 16-wide window of each partial map
  for (int it = tid; it < kQ * 8; it += kLossThreads) {
    const int r = it / 8, j0 = 4 * (it % 8);
    float out[3][4];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      float dv[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = j0 + 4 * q;
        if (col < kQs) {
          load4(s.d[c] + r * kQs + col, dv + 4 * q);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) dv[4 * q + e] = 0.f;
        }
      }
#pragma unroll
      for (int o = 0; o < 4; ++o) {
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t <= 2 * kR; ++t) acc = __fmaf_rn(w[t], dv[o + t], acc);
        out[c][o] = acc;
      }
    }
#pragma unroll
    for (int c = 0; c < 3; ++c)
      *reinterpret_cast<float4*>(s.a[c] + r * kOut + j0) = make_float4(out[c][0], out[c][1], out[c][2], out[c][3]);
  }
  __syncthreads();
  // 5. vertical adjoint (2 columns x 4 rows per item), L1 term, gradient out
  for (int it = tid; it < 16 * 8; it += kLossThreads) {
    const int j = 2 * (it % 16), i0 = 4 * (it / 16);
    float acc[3][4][2];
#pragma unroll
    for (int c = 0; c < 3; ++c)
#pragma unroll
      for (int o = 0; o < 4; ++o) acc[c][o][0] = acc[c][o][1] = 0.f;
#pragma unroll
    for (int rr = 0; rr < 14; ++rr) {
      const int row = i0 + rr;
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        const float2 av = *reinterpret_cast<const float2*>(s.a[c] + row * kOut + j);
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const int t = rr - o;
          if (t >= 0 && t <= 2 * kR) {
            acc[c][o][0] = __fmaf_rn(w[t], av.x, acc[c][o][0]);
            acc[c][o][1] = __fmaf_rn(w[t], av.y, acc[c][o][1]);
          }
        }
      }
    }
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = i0 + o, jj = j + e;
        const int gy = y0 + i, gx = x0 + jj;
        if (gy >= H || gx >= W) continue;
        const float xv = s.x[(i + 2 * kR) * kIn + jj + 2 * kR];
        const float yv = s.y[(i + 2 * kR) * kIn + jj + 2 * kR];
        const float r = xv - yv;
        l1_acc += fabsf(r);
        if (a.dx) {
          const float G = acc[0][o][e] + 2.f * xv * acc[1][o][e] + yv * acc[2][o][e];
          const float sgn = r > 0.f ? 1.f : (r < 0.f ? -1.f : 0.f);
          a.dx[ch * HW + static_cast<int64_t>(gy) * W + gx] = (1.f - a.lambda) * inv * sgn - a.lambda * inv * G;
        }
      }
  }

  // Block partial sums in float64, then the last CTA reduces all in fixed order.
  double l1 = l1_acc, ss = ssim_acc;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if (lane == 0) {
    s.red[0][warp] = l1;
    s.red[1][warp] = ss;
  }
  __syncthreads();
  const int nblocks = gridDim.x * gridDim.y * gridDim.z;
  const int bid = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  if (tid == 0) {
    double t0 = 0.0, t1 = 0.0;
    for (int k = 0; k < kLossThreads / 32; ++k) {
      t0 += s.red[0][k];
      t1 += s.red[1][k];
    }
    a.partials[2 * bid] = t0;
    a.partials[2 * bid + 1] = t1;
    __threadfence();
    const uint32_t ticket = atomicAdd(a.counter, 1u);
    s.last = ticket == static_cast<uint32_t>(nblocks - 1);
  }
  __syncthreads();
  if (!s.last) return;
  __threadfence();
  double p0 = 0.0, p1 = 0.0;
  for (int b = tid; b < nblocks; b += kLossThreads) {
    p0 += __ldcg(a.partials + 2 * b);
    p1 += __ldcg(a.partials + 2 * b + 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    p0 += __shfl_xor_sync(0xffffffffu, p0, o);
    p1 += __shfl_xor_sync(0xffffffffu, p1, o);
  }
  __syncthreads();
  if (lane == 0) {
    s.red[0][warp] = p0;
    s.red[1][warp] = p1;
  }
  __syncthreads();
  if (tid == 0) {
    double t0 = 0.0, t1 = 0.0;
    for (int k = 0; k < kLossThreads / 32; ++k) {
      t0 += s.red[0][k];
      t1 += s.red[1][k];
    }
    const double n3 = 3.0 * static_cast<double>(HW);
    const double l1m = t0 / n3, ssim = t1 / n3;
    a.out[0] = (1.0 - a.lambda) * l1m + a.lambda * (1.0 - ssim);
    a.out[1] = l1m;
    a.out[2] = ssim;
    *a.counter = 0u;  // ready for the next call
  }
}

}  // namespace

cudaError_t launch_loss(const LossArgs& a, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(loss_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sizeof(LossSmem)));
  if (e != cudaSuccess) return e;
  dim3 grid((a.width + kOut - 1) / kOut, (a.height + kOut - 1) / kOut, 3);
  loss_kernel<<<grid, kLossThreads, sizeof(LossSmem), st>>>(a);
  return cudaGetLastError();
}

int64_t loss_num_blocks(int height, int width) {
  return 3 * static_cast<int64_t>((width + kOut - 1) / kOut) * ((height + kOut - 1) / kOut);
}

}  // namespace gs
