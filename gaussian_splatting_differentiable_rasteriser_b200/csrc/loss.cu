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
// B200 design: one CTA per 32x32 output tile does everything in shared memory
// with halo recompute - no intermediate maps in HBM, so the kernel reads the
// two images once and writes the gradient once (36 B per pixel). Per channel:
// load the 52x52 input region (zero outside the image), separable 11-tap
// horizontal then vertical filtering of the 5 moments over the 42x42 region of
// SSIM-map positions the tile's gradient depends on, the map and its three
// partial derivatives there (zero outside the image), then the separable
// adjoint filter back onto the 32x32 tile. Block partial sums of |x - y| and
// of the map go to a small array that the last CTA to finish reduces in a
// fixed order in float64, so the loss is deterministic.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kOut = 32;                 // output tile side
constexpr int kR = 5;                    // window radius
constexpr int kQ = kOut + 2 * kR;        // 42: SSIM-map positions needed
constexpr int kIn = kOut + 4 * kR;       // 52: input pixels needed
constexpr int kLossThreads = 256;

struct LossSmem {
  float x[kIn * kIn];
  float y[kIn * kIn];
  float h[5][kIn * kQ];   // horizontal moments: rows of the input region, map columns
  float d[3][kQ * kQ];    // map partials dS/dmu_x, dS/dE[x^2], dS/dE[xy]
  float a[3][kQ * kOut];  // horizontally filtered partials: map rows, output columns
  double red[2][kLossThreads / 32];
  int last;
};

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

  for (int ch = 0; ch < 3; ++ch) {
    const float* X = a.x + ch * HW;
    const float* Yc = a.y + ch * HW;
    // 1. input region [y0 - 10, y0 + 42) x [x0 - 10, x0 + 42), zero padded
    for (int k = tid; k < kIn * kIn; k += kLossThreads) {
      const int r = k / kIn, c = k % kIn;
      const int gy = y0 - 2 * kR + r, gx = x0 - 2 * kR + c;
      const bool in = gy >= 0 && gy < H && gx >= 0 && gx < W;
      const int64_t g = static_cast<int64_t>(gy) * W + gx;
      s.x[k] = in ? X[g] : 0.0f;
      s.y[k] = in ? Yc[g] : 0.0f;
    }
    __syncthreads();
    // 2. horizontal pass of the five moments; map column j <-> image x0 - 5 + j
    for (int k = tid; k < kIn * kQ; k += kLossThreads) {
      const int r = k / kQ, j = k % kQ;
      const float* xr = s.x + r * kIn + j;
      const float* yr = s.y + r * kIn + j;
      float mx = 0.f, my = 0.f, mxx = 0.f, myy = 0.f, mxy = 0.f;
#pragma unroll
      for (int t = 0; t <= 2 * kR; ++t) {
        const float w = a.window[t], xv = xr[t], yv = yr[t];
        const float wx = w * xv, wy = w * yv;
        mx += wx;
        my += wy;
        mxx = __fmaf_rn(wx, xv, mxx);
        myy = __fmaf_rn(wy, yv, myy);
        mxy = __fmaf_rn(wx, yv, mxy);
      }
      s.h[0][k] = mx;
      s.h[1][k] = my;
      s.h[2][k] = mxx;
      s.h[3][k] = myy;
      s.h[4][k] = mxy;
    }
    __syncthreads();
    // 3. vertical pass, SSIM map and its partial derivatives at the 42x42 positions
    for (int k = tid; k < kQ * kQ; k += kLossThreads) {
      const int qi = k / kQ, qj = k % kQ;
      float m[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t <= 2 * kR; ++t) {
        const float w = a.window[t];
        const int o = (qi + t) * kQ + qj;
#pragma unroll
        for (int c = 0; c < 5; ++c) m[c] = __fmaf_rn(w, s.h[c][o], m[c]);
      }
      const int gy = y0 - kR + qi, gx = x0 - kR + qj;
      float dm = 0.f, dxx = 0.f, dxy = 0.f;
      if (gy >= 0 && gy < H && gx >= 0 && gx < W) {
        const float mux = m[0], muy = m[1];
        const float sxx = m[2] - mux * mux, syy = m[3] - muy * muy, sxy = m[4] - mux * muy;
        const float A1 = 2.f * mux * muy + C1, A2 = 2.f * sxy + C2;
        const float B1 = mux * mux + muy * muy + C1, B2 = sxx + syy + C2;
        const float iB = 1.0f / (B1 * B2);
        const float S = A1 * A2 * iB;
        // partials with mu_y, E[y^2] fixed: sxx = E[x^2] - mux^2, sxy = E[xy] - mux muy
        dm = (2.f * muy * A2 - 2.f * muy * A1) * iB - S * (2.f * mux / B1 - 2.f * mux / B2);
        dxx = -S / B2;
        dxy = 2.f * A1 * iB;
        if (qi >= kR && qi < kR + kOut && qj >= kR && qj < kR + kOut) ssim_acc += S;
      }
      s.d[0][k] = dm;
      s.d[1][k] = dxx;
      s.d[2][k] = dxy;
    }
    __syncthreads();
    // 4. horizontal adjoint onto the output columns (the window is symmetric)
    for (int k = tid; k < kQ * kOut; k += kLossThreads) {
      const int r = k / kOut, j = k % kOut;
      float acc[3] = {0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t <= 2 * kR; ++t) {
        const float w = a.window[t];
        const int o = r * kQ + j + t;
#pragma unroll
        for (int c = 0; c < 3; ++c) acc[c] = __fmaf_rn(w, s.d[c][o], acc[c]);
      }
      s.a[0][k] = acc[0];
      s.a[1][k] = acc[1];
      s.a[2][k] = acc[2];
    }
    __syncthreads();
    // 5. vertical adjoint, L1 term, gradient out
    for (int k = tid; k < kOut * kOut; k += kLossThreads) {
      const int i = k / kOut, j = k % kOut;
      const int gy = y0 + i, gx = x0 + j;
      if (gy >= H || gx >= W) continue;
      float acc[3] = {0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t <= 2 * kR; ++t) {
        const float w = a.window[t];
        const int o = (i + t) * kOut + j;
#pragma unroll
        for (int c = 0; c < 3; ++c) acc[c] = __fmaf_rn(w, s.a[c][o], acc[c]);
      }
      const float xv = s.x[(i + 2 * kR) * kIn + j + 2 * kR];
      const float yv = s.y[(i + 2 * kR) * kIn + j + 2 * kR];
      const float r = xv - yv;
      l1_acc += fabsf(r);
      if (a.dx) {
        const float G = acc[0] + 2.f * xv * acc[1] + yv * acc[2];
        const float sgn = r > 0.f ? 1.f : (r < 0.f ? -1.f : 0.f);
        a.dx[ch * HW + static_cast<int64_t>(gy) * W + gx] =
            (1.f - a.lambda) * inv * sgn - a.lambda * inv * G;
      }
    }
    __syncthreads();
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
  const int nblocks = gridDim.x * gridDim.y;
  const int bid = blockIdx.y * gridDim.x + blockIdx.x;
  if (tid == 0) {
    double t0 = 0.0, t1 = 0.0;
    for (int w = 0; w < kLossThreads / 32; ++w) {
      t0 += s.red[0][w];
      t1 += s.red[1][w];
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
    for (int w = 0; w < kLossThreads / 32; ++w) {
      t0 += s.red[0][w];
      t1 += s.red[1][w];
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
  dim3 grid((a.width + kOut - 1) / kOut, (a.height + kOut - 1) / kOut);
  loss_kernel<<<grid, kLossThreads, sizeof(LossSmem), st>>>(a);
  return cudaGetLastError();
}

int64_t loss_num_blocks(int height, int width) {
  return static_cast<int64_t>((width + kOut - 1) / kOut) * ((height + kOut - 1) / kOut);
}

}  // namespace gs
