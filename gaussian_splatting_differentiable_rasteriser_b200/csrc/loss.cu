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
// B200 design: one CTA per channel and 32-column x kStrip-row strip walks down
// the strip in steps of 16 rows, with the separable filters pipelined through
// ring buffers in shared memory, so every input row is filtered horizontally
// once, every SSIM-map row is formed once, and every intermediate stays on
// chip (the kernel reads the two images once and writes the gradient once, 36
// B per pixel over the three channels). A step:
//   1. loads 16 input rows x 52 columns of both images (zero outside);
//   2. filters them horizontally into the 5 moments at the 42 map columns
//      the strip's gradient depends on (ring of 28 rows);
//   3. filters 16 map rows vertically from the ring, forms the SSIM map and
//      its partial derivatives there (zero outside the image);
//   4. filters those partials horizontally onto the 32 output columns (ring);
//   5. filters the output rows whose 11 rows of partials are complete
//      vertically and writes dL/dx with the L1 term.
// Each stage lags the previous one by the window radius, so the outputs of a
// step are 20 rows behind its inputs. Block partial sums of |x - y| and of the
// map go to a small array that the last CTA to finish reduces in a fixed
// order in float64, so the loss is deterministic.
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kCols = kLossCols;          // output columns per CTA
constexpr int kStrip = kLossStrip;        // output rows per CTA
constexpr int kStep = 16;                 // rows per pipeline step
constexpr int kR = 5;                     // window radius
constexpr int kMapCols = kCols + 2 * kR;  // 42: SSIM-map columns needed
constexpr int kInCols = kCols + 4 * kR;   // 52: input columns needed
constexpr int kInS = 56;                  // padded input row stride (zeros beyond 52)
constexpr int kHs = 44;                   // padded map row stride (16-byte rows)
constexpr int kRing = 28;                 // ring rows (>= kStep + 2 kR = 26)
constexpr int kLossThreads = 256;
static_assert(kRing >= kStep + 2 * kR, "a ring must hold a step and its halo");

// Ring slot of a row given its offset from the strip's first ring row
// (offsets down to -2 kRing occur for rows above the strip, which are never read).
__device__ __forceinline__ int ring_slot(int v) { return (v + 2 * kRing) % kRing; }

struct LossSmem {
  float in[2][kStep][kInS];       // x, y rows of this step
  float h[5][kRing][kHs];         // horizontal moments mu_x, mu_y, E[x^2], E[y^2], E[xy]
  float d[3][kStep][kHs];         // map partials dS/dmu_x, dS/dE[x^2], dS/dE[xy] of this step
  float a[3][kRing][kCols];       // horizontally filtered partials
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

constexpr int kLoadsPerThread = (2 * kStep * kInS + kLossThreads - 1) / kLossThreads;  // 7

// The input rows [hb, hb + kStep) x image columns [x0 - 2 kR, x0 - 2 kR + kInS)
// of both images, as they lie in LossSmem::in, this thread's share (zero
// outside the image, beyond the 52 needed columns and beyond the rows the
// strip needs).
__device__ __forceinline__ void load_rows(const LossArgs& a, const float* X, const float* Yc, int x0, int hb,
                                          int Yend, int tid, float (&pre)[kLoadsPerThread]) {
  const int H = a.height, W = a.width;
#pragma unroll
  for (int u = 0; u < kLoadsPerThread; ++u) {
    const int k = tid + u * kLossThreads;
    const int img = k / (kStep * kInS), rem = k % (kStep * kInS);
    const int r = rem / kInS, c = rem % kInS;
    const int gy = hb + r, gx = x0 - 2 * kR + c;
    const bool in = k < 2 * kStep * kInS && c < kInCols && gy >= 0 && gy < H && gy < Yend + 2 * kR &&
                    gx >= 0 && gx < W;
    pre[u] = in ? __ldg((img ? Yc : X) + static_cast<int64_t>(gy) * W + gx) : 0.0f;
  }
}

__global__ void __launch_bounds__(kLossThreads, 4) loss_kernel(LossArgs a) {
  chain_wait();
  chain_release();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  LossSmem& s = *reinterpret_cast<LossSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int x0 = blockIdx.x * kCols, Y0 = blockIdx.y * kStrip;
  const int H = a.height, W = a.width;
  const int Yend = min(Y0 + kStrip, H);
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

  // outputs trail the inputs by 4 kR rows: step st writes output rows
  // [Y0 - 4 kR + kStep st, Y0 - 4 kR + kStep (st + 1)), so L rows need the
  // smallest S with kStep (S - 1) >= L + 4 kR - kStep
  const int steps = (Yend - Y0 + 4 * kR - 1) / kStep + 1;
  float pre[kLoadsPerThread];
  for (int st = 0; st < steps; ++st) {
    const int hb = Y0 - 2 * kR + kStep * st;  // first input row of this step
    const int mb = hb - kR;                   // first map row of this step
    const int ob = mb - kR;                   // first output row of this step
    // 1. input rows [hb, hb + 16) x image columns [x0 - 10, x0 + 46) (zero
    //    outside), loaded into registers one step ahead so their latency
    //    overlaps the previous step's filtering
    if (st == 0) load_rows(a, X, Yc, x0, hb, Yend, tid, pre);
#pragma unroll
    for (int u = 0; u < kLoadsPerThread; ++u) {
      const int k = tid + u * kLossThreads;
      if (k < 2 * kStep * kInS) (&s.in[0][0][0])[k] = pre[u];
    }
    __syncthreads();
    if (st + 1 < steps) load_rows(a, X, Yc, x0, hb + kStep, Yend, tid, pre);
    // 2. horizontal moments of the 16 rows at map columns j (image x0 - 5 + j),
    //    4 columns per item from a 14-wide window held in registers
    for (int it = tid; it < kStep * 11; it += kLossThreads) {
      const int r = it / 11, j0 = 4 * (it % 11);
      float xv[16], yv[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        load4(&s.in[0][r][j0 + 4 * q], xv + 4 * q);  // j0 + 4 q + 3 <= 55 < kInS
        load4(&s.in[1][r][j0 + 4 * q], yv + 4 * q);
      }
      float pxx[14], pyy[14], pxy[14];
#pragma unroll
      for (int e = 0; e < 14; ++e) {
        pxx[e] = xv[e] * xv[e];
        pyy[e] = yv[e] * yv[e];
        pxy[e] = xv[e] * yv[e];
      }
      const int ring = ring_slot(hb + r - Y0 + 2 * kR);
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
        *reinterpret_cast<float4*>(&s.h[c][ring][j0]) = make_float4(m[c][0], m[c][1], m[c][2], m[c][3]);
    }
    __syncthreads();
    // 3. vertical pass for map rows [mb, mb + 16) (1 column x 4 rows per item),
    //    SSIM map and its partial derivatives
    for (int it = tid; it < kMapCols * 4; it += kLossThreads) {
      const int j = it % kMapCols, k0 = 4 * (it / kMapCols);
      const int q0 = mb + k0;
      float acc[5][4];
#pragma unroll
      for (int c = 0; c < 5; ++c)
#pragma unroll
        for (int o = 0; o < 4; ++o) acc[c][o] = 0.f;
      if (q0 + 3 >= Y0 - kR) {  // rows above Y0 - 5 feed no output of this strip
        int ring = ring_slot(q0 - kR - Y0 + 2 * kR);  // advanced one row at a time below
#pragma unroll
        for (int rr = 0; rr < 14; ++rr) {
#pragma unroll
          for (int c = 0; c < 5; ++c) {
            const float hv = s.h[c][ring][j];
#pragma unroll
            for (int o = 0; o < 4; ++o) {
              const int t = rr - o;
              if (t >= 0 && t <= 2 * kR) acc[c][o] = __fmaf_rn(w[t], hv, acc[c][o]);
            }
          }
          ring = ring + 1 == kRing ? 0 : ring + 1;
        }
      }
#pragma unroll
      for (int o = 0; o < 4; ++o) {
        const int q = q0 + o, gx = x0 - kR + j;
        float dm = 0.f, dxx = 0.f, dxy = 0.f;
        if (q >= 0 && q < H && q >= Y0 - kR && gx >= 0 && gx < W) {
          const float mux = acc[0][o], muy = acc[1][o];
          const float sxx = acc[2][o] - mux * mux, syy = acc[3][o] - muy * muy;
          const float sxy = acc[4][o] - mux * muy;
          const float A1 = 2.f * mux * muy + C1, A2 = 2.f * sxy + C2;
          const float B1 = mux * mux + muy * muy + C1, B2 = sxx + syy + C2;
          // B1 >= C1 and B2 >= C2 > 0: the fast reciprocal is accurate to a few ulp here
          const float iB1 = __fdividef(1.0f, B1), iB2 = __fdividef(1.0f, B2);
          const float iB = iB1 * iB2;
          const float S = A1 * A2 * iB;
          // partials with mu_y, E[y^2] fixed: sxx = E[x^2] - mux^2, sxy = E[xy] - mux muy
          dm = 2.f * muy * (A2 - A1) * iB - 2.f * mux * S * (iB1 - iB2);
          dxx = -S * iB2;
          dxy = 2.f * A1 * iB;
          if (q >= Y0 && q < Yend && j >= kR && j < kR + kCols) ssim_acc += S;
        }
        s.d[0][k0 + o][j] = dm;
        s.d[1][k0 + o][j] = dxx;
        s.d[2][k0 + o][j] = dxy;
      }
    }
    __syncthreads();
    // 4. horizontal adjoint of the map rows onto the 32 output columns
    //    (the window is symmetric), 2 columns per item
    for (int it = tid; it < kStep * (kCols / 2); it += kLossThreads) {
      const int k = it / (kCols / 2), jj = 2 * (it % (kCols / 2));
      const int ring = ring_slot(mb + k - Y0 + kR);
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        float dv[12];
#pragma unroll
        for (int e = 0; e < 12; e += 2) {
          const float2 t2 = *reinterpret_cast<const float2*>(&s.d[c][k][jj + e]);
          dv[e] = t2.x;
          dv[e + 1] = t2.y;
        }
        float o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int t = 0; t <= 2 * kR; ++t) {
          o0 = __fmaf_rn(w[t], dv[t], o0);
          o1 = __fmaf_rn(w[t], dv[t + 1], o1);
        }
        *reinterpret_cast<float2*>(&s.a[c][ring][jj]) = make_float2(o0, o1);
      }
    }
    __syncthreads();
    // 5. vertical adjoint for output rows [ob, ob + 16) (1 column x 2 rows per item),
    //    L1 term and the gradient
    for (int it = tid; it < kCols * (kStep / 2); it += kLossThreads) {
      const int jj = it % kCols, k0 = 2 * (it / kCols);
      const int r0 = ob + k0;
      if (r0 + 1 < Y0 || r0 >= Yend) continue;
      float acc[3][2];
#pragma unroll
      for (int c = 0; c < 3; ++c) acc[c][0] = acc[c][1] = 0.f;
      int ring = ring_slot(r0 - kR - Y0 + kR);  // advanced one row at a time below
#pragma unroll
      for (int rr = 0; rr < 12; ++rr) {
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          const float av = s.a[c][ring][jj];
#pragma unroll
          for (int o = 0; o < 2; ++o) {
            const int t = rr - o;
            if (t >= 0 && t <= 2 * kR) acc[c][o] = __fmaf_rn(w[t], av, acc[c][o]);
          }
        }
        ring = ring + 1 == kRing ? 0 : ring + 1;
      }
      const int gx = x0 + jj;
#pragma unroll
      for (int o = 0; o < 2; ++o) {
        const int gy = r0 + o;
        if (gy < Y0 || gy >= Yend || gx >= W) continue;
        const int64_t g = static_cast<int64_t>(gy) * W + gx;
        const float xv = __ldg(X + g), yv = __ldg(Yc + g);
        const float r = xv - yv;
        l1_acc += fabsf(r);
        if (a.dx) {
          const float G = acc[0][o] + 2.f * xv * acc[1][o] + yv * acc[2][o];
          const float sgn = r > 0.f ? 1.f : (r < 0.f ? -1.f : 0.f);
          a.dx[ch * HW + g] = (1.f - a.lambda) * inv * sgn - a.lambda * inv * G;
        }
      }
    }
    // the next step's stage 1 writes only the input rows; its stage 2 waits at a barrier
  }
  __syncthreads();

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
  dim3 grid((a.width + kCols - 1) / kCols, (a.height + kStrip - 1) / kStrip, 3);
  return launch_chained(loss_kernel, grid, dim3(kLossThreads), sizeof(LossSmem), st, a);
}

int64_t loss_num_blocks(int height, int width) { return loss_blocks(height, width); }

}  // namespace gs
