// Preprocess: one thread per Gaussian projects it to the screen.
//
// Method: "Gaussian splatting training" study notes (bailiping.com), slides on
// the parametrisation and "J is the 2 x 3 Jacobian of perspective projection";
// "How a computer rebuilds a real place ... Gaussian Splats" (taosengine.com),
// sections "Flattening a 3D blob into a 2D oval (EWA projection)" (T = J W,
// Sigma' = T Sigma T^T, conic, radius from the largest eigenvalue, tile rect)
// and "Spherical harmonics: color that changes with viewing angle".
//
// B200 notes: the kernel is HBM-bound (236 B of parameters in, 48 + 17 B out
// per Gaussian at SH degree 3). Each CTA stages its Gaussians' parameter
// planes in shared memory with bulk asynchronous copies (the untiled TMA
// path) completed on an mbarrier, then computes from shared memory. The geometry runs in float64 - free next to the memory time - so that
// the integer decisions taken from it (culling, tile rect, depth key) are
// stable to ~1e-15 and do not depend on float32 rounding order.
#include "bulk_copy.cuh"
#include "gs_kernels.cuh"
#include "sh.cuh"

namespace gs {

namespace {

__device__ __forceinline__ double dot3(const double* a, const double* b) {
  return a[0] * b[0] + a[1] * b[1] + a[2] * b[2];
}

constexpr int kPreThreads = 256;
constexpr int kGeomPlanes = 11;  // means 3, log-scales 3, quats 4, opacity logit 1

// The parameters of a CTA's 256 Gaussians, one 1 KB row per plane: the
// geometric planes, then the 3 x (kDeg + 1)^2 active SH planes.
template <int kDeg>
struct PreprocessSmem {
  float plane[kGeomPlanes + 3 * (kDeg + 1) * (kDeg + 1)][kPreThreads];
  uint64_t bar[2];  // geometry planes, SH planes
};

template <int kDeg>
__global__ void __launch_bounds__(kPreThreads, 3) preprocess_kernel(PreprocessArgs a) {
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
  constexpr int kPlanes = kGeomPlanes + 3 * nk;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  PreprocessSmem<kDeg>& sm = *reinterpret_cast<PreprocessSmem<kDeg>*>(smem_raw);
  const int tid = threadIdx.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kPreThreads;
  const int64_t i = i0 + tid;
  const int64_t np = a.n_pad;
  // Stage the CTA's slice of every parameter plane in shared memory with bulk
  // asynchronous copies issued by one thread, so all of a Gaussian's loads
  // (about 240 B at degree 3) are in flight at once instead of behind the
  // geometry's dependency chain. The 11 geometry planes complete on one
  // mbarrier and the SH planes on another: the float64 geometry runs while the
  // SH planes are still arriving. Planes start 16-byte aligned (n_pad % 4 == 0,
  // 16-byte aligned parameter pointers) and a slice is a multiple of 4 floats.
  if (tid == 0) {
    mbar_init(&sm.bar[0]);
    mbar_init(&sm.bar[1]);
    const int cnt = static_cast<int>(np - i0 < kPreThreads ? np - i0 : kPreThreads);
    const uint32_t bytes = static_cast<uint32_t>(cnt) * 4u;
    mbar_arrive_expect_tx(&sm.bar[0], bytes * kGeomPlanes);
#pragma unroll
    for (int c = 0; c < 3; ++c) bulk_copy_g2s(sm.plane[c], a.means + c * np + i0, bytes, &sm.bar[0]);
#pragma unroll
    for (int c = 0; c < 3; ++c) bulk_copy_g2s(sm.plane[3 + c], a.log_scales + c * np + i0, bytes, &sm.bar[0]);
#pragma unroll
    for (int c = 0; c < 4; ++c) bulk_copy_g2s(sm.plane[6 + c], a.quats + c * np + i0, bytes, &sm.bar[0]);
    bulk_copy_g2s(sm.plane[10], a.opacity_logits + i0, bytes, &sm.bar[0]);
    mbar_arrive_expect_tx(&sm.bar[1], bytes * (kPlanes - kGeomPlanes));
    for (int ch = 0; ch < 3; ++ch)
      for (int k = 0; k < nk; ++k)
        bulk_copy_g2s(sm.plane[kGeomPlanes + ch * nk + k],
                      a.sh + (static_cast<int64_t>(ch) * a.sh_k + k) * np + i0, bytes, &sm.bar[1]);
  }
  __syncthreads();  // the barriers are initialised before anyone waits on them
  // Every thread waits for the geometry planes itself (bounded); thread 0
  // records a timeout and, before the CTA can retire, waits for all copies.
  bool ok = mbar_wait(&sm.bar[0], 0, 1 << 16);
  if (!__syncthreads_and(ok)) {
    if (tid == 0) {
      // Nothing computed from this slice is used (the error fails the
      // launch), but the CTA must not retire before its copies have landed.
      record_error(a.err, kErrCopyTimeout);
      mbar_drain(&sm.bar[0], 0, 2000000);
      mbar_drain(&sm.bar[1], 0, 2000000);
    }
    __syncthreads();
    if (i < a.n) {  // parameters not staged: treat as culled
      a.screen[i] = Screen{};
      a.depth[i] = 0.0f;
      a.rect[i] = make_uint2(1u, 1u);
      a.touched[i] = 0u;
      a.clamped[i] = 0u;
    }
    if (tid == 0) a.block_sums[blockIdx.x] = make_uint2(0u, 0u);
    return;
  }
  uint32_t touched = 0;
  uint32_t dkey = 0;
  bool visible = false;
  bool sh_ok = true;  // the SH planes arrived (waited for where colour is needed)
  if (i < a.n) {
    const CamArgs& cam = a.cam;
    const double p[3] = {sm.plane[0][tid], sm.plane[1][tid], sm.plane[2][tid]};
    // p_c = R p + t, each row summed left to right without fused multiply-add:
    // the depth key float32(Z) is then the same on every implementation.
    double pc[3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
      pc[r] = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(cam.R[3 * r], p[0]),
                                            __dmul_rn(cam.R[3 * r + 1], p[1])),
                                  __dmul_rn(cam.R[3 * r + 2], p[2])),
                        static_cast<double>(cam.t[r]));
    const double X = pc[0], Y = pc[1], Z = pc[2];
    const float depth = __double2float_rn(Z);
    Screen s;
    s.a = make_float4(0.f, 0.f, 0.f, 0.f);
    s.b = s.a;
    s.c = s.a;
    uint2 rect = make_uint2(1u, 1u);  // x0 = 1 > x1 = 0: empty
    uint8_t clamped = 0;
    if (Z > static_cast<double>(cam.near_z)) {
      // Sigma = M M^T, M = R(q/|q|) diag(exp(ls))
      const double qw = sm.plane[6][tid], qx = sm.plane[7][tid], qy = sm.plane[8][tid],
                   qz = sm.plane[9][tid];
      const double qn = sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
      const double w = qw / qn, x = qx / qn, y = qy / qn, z = qz / qn;
      const double Rq[9] = {1.0 - 2.0 * (y * y + z * z), 2.0 * (x * y - w * z), 2.0 * (x * z + w * y),
                            2.0 * (x * y + w * z), 1.0 - 2.0 * (x * x + z * z), 2.0 * (y * z - w * x),
                            2.0 * (x * z - w * y), 2.0 * (y * z + w * x), 1.0 - 2.0 * (x * x + y * y)};
      const double sc[3] = {exp(static_cast<double>(sm.plane[3][tid])),
                            exp(static_cast<double>(sm.plane[4][tid])),
                            exp(static_cast<double>(sm.plane[5][tid]))};
      double M[9];
#pragma unroll
      for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int c = 0; c < 3; ++c) M[3 * r + c] = Rq[3 * r + c] * sc[c];
      const double S00 = dot3(M, M), S01 = dot3(M, M + 3), S02 = dot3(M, M + 6);
      const double S11 = dot3(M + 3, M + 3), S12 = dot3(M + 3, M + 6), S22 = dot3(M + 6, M + 6);
      // T = J W (rows t0, t1)
      const double iz = 1.0 / Z;
      const double jx = cam.fx * iz, jy = cam.fy * iz;
      const double jxz = -cam.fx * X * iz * iz, jyz = -cam.fy * Y * iz * iz;
      double t0[3], t1[3];
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        t0[c] = jx * cam.R[c] + jxz * cam.R[6 + c];
        t1[c] = jy * cam.R[3 + c] + jyz * cam.R[6 + c];
      }
      // Sigma' = T Sigma T^T + 0.3 I
      const double u0[3] = {S00 * t0[0] + S01 * t0[1] + S02 * t0[2],
                            S01 * t0[0] + S11 * t0[1] + S12 * t0[2],
                            S02 * t0[0] + S12 * t0[1] + S22 * t0[2]};
      const double u1[3] = {S00 * t1[0] + S01 * t1[1] + S02 * t1[2],
                            S01 * t1[0] + S11 * t1[1] + S12 * t1[2],
                            S02 * t1[0] + S12 * t1[1] + S22 * t1[2]};
      const double ca = dot3(t0, u0) + kDilation;
      const double cb = dot3(t0, u1);
      const double cc = dot3(t1, u1) + kDilation;
      const double det = ca * cc - cb * cb;
      // Mip-Splatting compensation: sqrt(det V / det(V + 0.3 I)), V undilated
      double comp = 1.0;
      if (a.mip_comp) {
        const double det0 = (ca - kDilation) * (cc - kDilation) - cb * cb;
        comp = det0 > 0.0 ? sqrt(det0 / det) : 0.0;
      }
      if (det > 0.0) {
        const double u = cam.fx * X * iz + cam.cx;
        const double v = cam.fy * Y * iz + cam.cy;
        const double mid = 0.5 * (ca + cc);
        const double lmax = mid + sqrt(fmax(mid * mid - det, 0.0));
        double rad = kRadiusSigmas * sqrt(lmax);
        if (a.opacity_rect) {
          // opacity-aware cut: beyond sqrt(2 E) sigma along the long axis alpha < 1/255
          const double od = 1.0 / (1.0 + exp(-static_cast<double>(sm.plane[10][tid]))) * comp;
          const double e_cut = fmin(4.5, log(fmax(od * 255.0, 1.0001)));
          rad = sqrt(2.0 * e_cut) * sqrt(lmax);
        }
        // tiles whose pixels [16 t, 16 t + 15] meet [u - r, u + r] (same for y)
        double fx0 = fmax(ceil((u - rad - (kTile - 1)) / kTile), 0.0);
        double fx1 = fmin(floor((u + rad) / kTile), static_cast<double>(cam.tiles_x - 1));
        double fy0 = fmax(ceil((v - rad - (kTile - 1)) / kTile), 0.0);
        double fy1 = fmin(floor((v + rad) / kTile), static_cast<double>(cam.tiles_y - 1));
        if (fx0 <= fx1 && fy0 <= fy1) {  // false for NaN too
          const uint32_t x0 = static_cast<uint32_t>(fx0), x1 = static_cast<uint32_t>(fx1);
          const uint32_t y0 = static_cast<uint32_t>(fy0), y1 = static_cast<uint32_t>(fy1);
          rect = make_uint2(x0 | (x1 << 16), y0 | (y1 << 16));
          touched = (x1 - x0 + 1) * (y1 - y0 + 1);
          visible = true;
          dkey = __float_as_uint(depth);
          float opacity = 1.0f / (1.0f + expf(-sm.plane[10][tid]));
          if (a.mip_comp) opacity = static_cast<float>(static_cast<double>(opacity) * comp);
          // view-dependent colour at v = normalize(p - campos); its SH planes
          // were still arriving while the geometry above ran
          sh_ok = mbar_wait(&sm.bar[1], 0, 1 << 16);
          double d[3] = {p[0] - cam.campos[0], p[1] - cam.campos[1], p[2] - cam.campos[2]};
          const double dn = sqrt(dot3(d, d));
          const float dx = static_cast<float>(d[0] / dn), dy = static_cast<float>(d[1] / dn),
                      dz = static_cast<float>(d[2] / dn);
          float Yk[16];
          sh_basis(kDeg, dx, dy, dz, Yk);
          float rgb[3];
#pragma unroll
          for (int ch = 0; ch < 3; ++ch) {
            float col = 0.0f;
#pragma unroll
            for (int k = 0; k < nk; ++k) col = fmaf(sm.plane[kGeomPlanes + ch * nk + k][tid], Yk[k], col);
            if (col < 0.0f) {
              col = 0.0f;
              clamped |= static_cast<uint8_t>(1u << ch);
            }
            rgb[ch] = col;
          }
          // conic (cc, -cb, ca) / det in the exponent form, and the box of the
          // alpha >= 1/255 region: o exp(-e) >= 1/255 exactly when e <= E =
          // ln(255 o), an ellipse with axis-aligned half-widths sqrt(2 E a),
          // sqrt(2 E c) (a, c the diagonal of Sigma'), widened by 0.1% + 0.02 px so
          // float32 rounding of the per-pixel alpha never passes the floor outside.
          const double l2e = 1.4426950408889634;
          const double E = log(255.0 * static_cast<double>(opacity));
          float hx = -1.0f, hy = -1.0f;
          if (E > 0.0) {
            hx = static_cast<float>(sqrt(2.0 * E * ca) * 1.001 + 0.02);
            hy = static_cast<float>(sqrt(2.0 * E * cc) * 1.001 + 0.02);
          }
          s.a = make_float4(static_cast<float>(u), static_cast<float>(v),
                            static_cast<float>(-0.5 * l2e * cc / det), static_cast<float>(l2e * cb / det));
          s.b = make_float4(static_cast<float>(-0.5 * l2e * ca / det),
                            static_cast<float>(log2(static_cast<double>(opacity))), rgb[0], rgb[1]);
          s.c = make_float4(rgb[2], opacity, hx, hy);
        }
      }
    }
    if (!sh_ok) {  // the SH copies did not land in time: treat as culled
      s = Screen{};
      rect = make_uint2(1u, 1u);
      touched = 0u;
      clamped = 0u;
      visible = false;
      record_error(a.err, kErrCopyTimeout);
    }
    a.screen[i] = s;
    a.depth[i] = depth;
    a.rect[i] = rect;
    a.touched[i] = touched;
    a.clamped[i] = clamped;
  }
  // Before the CTA can retire, its SH copies must have landed even where no
  // thread needed them (every Gaussian of the slice culled).
  if (tid == 0 && !mbar_wait(&sm.bar[1], 0, 1 << 16)) {
    record_error(a.err, kErrCopyTimeout);
    mbar_drain(&sm.bar[1], 0, 2000000);
  }

  // Block totals of tiles touched and of visible Gaussians (for the entry
  // count and the compaction's prefix sum) and the depth-key range of visible
  // Gaussians (to size the depth sort's key).
  __shared__ uint32_t s_sum[8];
  __shared__ uint32_t s_vis[8];
  uint32_t t = touched;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  const uint32_t nvis = __popc(__ballot_sync(0xffffffffu, touched != 0u));
  uint32_t kmin = visible ? dkey : 0xffffffffu, kmax = visible ? dkey : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    s_sum[warp] = t;
    s_vis[warp] = nvis;
    if (kmin <= kmax) {
      atomicMin(&a.depth_range[0], kmin);
      atomicMax(&a.depth_range[1], kmax);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0, v = 0;
    for (int k = 0; k < (blockDim.x >> 5); ++k) {
      b += s_sum[k];
      v += s_vis[k];
    }
    a.block_sums[blockIdx.x] = make_uint2(b, v);
  }
}

// Exclusive prefix of the per-block visible counts (one CTA of 1024 threads),
// plus the entry and visible totals and the depth-key range copied into the
// readback record.
__global__ void __launch_bounds__(1024) scan_blocks_kernel(const uint2* block_sums, int64_t nb,
                                                           uint32_t* visible_prefix,
                                                           const uint32_t* depth_range,
                                                           ForwardInfo* info) {
  __shared__ uint64_t s_warp[32];
  __shared__ uint32_t s_vwarp[32];
  const int tid = threadIdx.x;
  const int64_t per = (nb + blockDim.x - 1) / blockDim.x;
  const int64_t lo = tid * per, hi = min(nb, lo + per);
  uint64_t entries = 0;
  uint32_t local = 0;
  for (int64_t k = lo; k < hi; ++k) {
    const uint2 b = block_sums[k];
    entries += b.x;
    local += b.y;
  }
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) entries += __shfl_xor_sync(0xffffffffu, entries, o);
  // inclusive scan of the visible counts across the CTA
  uint32_t v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) {
    s_vwarp[warp] = v;
    s_warp[warp] = entries;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t w = s_vwarp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    s_vwarp[lane] = w;
    uint64_t e = s_warp[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    if (lane == 0) s_warp[0] = e;
  }
  __syncthreads();
  uint32_t run = v - local + (warp > 0 ? s_vwarp[warp - 1] : 0u);
  for (int64_t k = lo; k < hi; ++k) {
    visible_prefix[k] = run;
    run += block_sums[k].y;
  }
  if (tid == 0) {
    info->num_entries = s_warp[0];
    info->num_visible = s_vwarp[31];
    info->depth_min = depth_range[0];
    info->depth_max = depth_range[1];
  }
}

template <int kDeg>
cudaError_t launch_preprocess_deg(const PreprocessArgs& a, unsigned grid, cudaStream_t st) {
  const int smem = static_cast<int>(sizeof(PreprocessSmem<kDeg>));
  cudaError_t e = cudaFuncSetAttribute(preprocess_kernel<kDeg>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  preprocess_kernel<kDeg><<<grid, kPreThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_preprocess(const PreprocessArgs& a, int64_t num_blocks, cudaStream_t st) {
  if (a.n == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>(num_blocks);
  switch (a.active_degree) {
    case 0: return launch_preprocess_deg<0>(a, grid, st);
    case 1: return launch_preprocess_deg<1>(a, grid, st);
    case 2: return launch_preprocess_deg<2>(a, grid, st);
    default: return launch_preprocess_deg<3>(a, grid, st);
  }
}

cudaError_t launch_scan_blocks(const uint2* block_sums, int64_t num_blocks, uint32_t* visible_prefix,
                               const uint32_t* depth_range, ForwardInfo* info, cudaStream_t st) {
  scan_blocks_kernel<<<1, 1024, 0, st>>>(block_sums, num_blocks, visible_prefix, depth_range, info);
  return cudaGetLastError();
}

}  // namespace gs
