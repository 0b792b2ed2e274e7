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
// path) completed on mbarriers, then computes from shared memory. The
// camera-space position and depth key are computed in float64 and the
// covariance chain in float32, redone in float64 where a tile bound lies near
// a tile boundary, so that the integer decisions taken from them (culling,
// tile rect, depth key) do not depend on float32 rounding.
#include "bulk_copy.cuh"
#include "gs_kernels.cuh"
#include "sh.cuh"

namespace gs {

namespace {

constexpr int kPreThreads = kGaussBlock;

// Screen covariance of one Gaussian before the dilation, V = T Sigma T^T with
// T = J W and Sigma = M M^T, M = R(q/|q|) diag(exp(ls)), computed in type S.
// With w_k = t0 . M_k and v_k = t1 . M_k (M_k the columns of M, t0 and t1 the
// rows of T): V = [[w.w, w.v], [w.v, v.v]] and det V = |w x v|^2 (Lagrange's
// identity), so det V and det(V + 0.3 I) = det V + 0.3 (V00 + V11) + 0.09 are
// sums of non-negative terms and carry no cancellation in float32.
template <typename S>
struct ScreenCov {
  S a0, b0, c0, det0;
};

template <typename S>
__device__ __forceinline__ ScreenCov<S> screen_cov(const float q4[4], const float ls3[3], double X, double Y,
                                                   double Z, const CamArgs& cam) {
  const S qw = q4[0], qx = q4[1], qy = q4[2], qz = q4[3];
  const S qn = sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
  const S w = qw / qn, x = qx / qn, y = qy / qn, z = qz / qn;
  const S one = 1, two = 2;
  const S Rq[9] = {one - two * (y * y + z * z), two * (x * y - w * z), two * (x * z + w * y),
                   two * (x * y + w * z), one - two * (x * x + z * z), two * (y * z - w * x),
                   two * (x * z - w * y), two * (y * z + w * x), one - two * (x * x + y * y)};
  const S sc[3] = {exp(static_cast<S>(ls3[0])), exp(static_cast<S>(ls3[1])), exp(static_cast<S>(ls3[2]))};
  const S iz = one / static_cast<S>(Z);
  const S fx = static_cast<S>(cam.fx), fy = static_cast<S>(cam.fy);
  const S jx = fx * iz, jy = fy * iz;
  const S jxz = -fx * static_cast<S>(X) * iz * iz, jyz = -fy * static_cast<S>(Y) * iz * iz;
  S t0[3], t1[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    t0[c] = jx * static_cast<S>(cam.R[c]) + jxz * static_cast<S>(cam.R[6 + c]);
    t1[c] = jy * static_cast<S>(cam.R[3 + c]) + jyz * static_cast<S>(cam.R[6 + c]);
  }
  S wv[3], vv[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    wv[k] = (t0[0] * Rq[k] + t0[1] * Rq[3 + k] + t0[2] * Rq[6 + k]) * sc[k];
    vv[k] = (t1[0] * Rq[k] + t1[1] * Rq[3 + k] + t1[2] * Rq[6 + k]) * sc[k];
  }
  ScreenCov<S> r;
  r.a0 = wv[0] * wv[0] + wv[1] * wv[1] + wv[2] * wv[2];
  r.b0 = wv[0] * vv[0] + wv[1] * vv[1] + wv[2] * vv[2];
  r.c0 = vv[0] * vv[0] + vv[1] * vv[1] + vv[2] * vv[2];
  const S cx = wv[1] * vv[2] - wv[2] * vv[1], cy = wv[2] * vv[0] - wv[0] * vv[2], cz = wv[0] * vv[1] - wv[1] * vv[0];
  r.det0 = cx * cx + cy * cy + cz * cz;
  return r;
}

// Tile-rect radius from the dilated covariance (the largest eigenvalue, with
// the cancellation-free discriminant) and, with the opacity-aware cut, the
// opacity o (times the compensation factor).
template <typename S>
__device__ __forceinline__ S rect_radius(const ScreenCov<S>& v, bool opacity_rect, S o) {
  const S a = v.a0 + static_cast<S>(kDilation), c = v.c0 + static_cast<S>(kDilation);
  const S hd = static_cast<S>(0.5) * (a - c);
  const S lmax = static_cast<S>(0.5) * (a + c) + sqrt(hd * hd + v.b0 * v.b0);
  if (!opacity_rect) return static_cast<S>(kRadiusSigmas) * sqrt(lmax);
  const S e_cut = fmin(static_cast<S>(4.5), log(fmax(o * static_cast<S>(255), static_cast<S>(1.0001))));
  return sqrt(static_cast<S>(2) * e_cut) * sqrt(lmax);
}

// The compensation factor sqrt(det V / det(V + 0.3 I)) (1 when not enabled).
template <typename S>
__device__ __forceinline__ S compensation(const ScreenCov<S>& v, bool on) {
  if (!on) return static_cast<S>(1);
  const S det = v.det0 + static_cast<S>(kDilation) * (v.a0 + v.c0) + static_cast<S>(kDilation * kDilation);
  return v.det0 > static_cast<S>(0) ? sqrt(v.det0 / det) : static_cast<S>(0);
}

// x is farther than m from every integer (the rounding of x by ceil or floor
// cannot change within +-m).
__device__ __forceinline__ bool clear_of_integers(double x, double m) { return fabs(x - rint(x)) > m; }
constexpr int kGeomPlanes = 11;  // means 3, log-scales 3, quats 4, opacity logit 1

// The parameters of a CTA's 256 Gaussians, one 1 KB row per plane: the
// geometric planes, then the 3 x (kDeg + 1)^2 active SH planes.
template <int kDeg>
struct PreprocessSmem {
  float plane[kGeomPlanes + 3 * (kDeg + 1) * (kDeg + 1)][kPreThreads];
  uint64_t bar[2];  // geometry planes, SH planes
};

template <int kDeg>
__global__ void __launch_bounds__(kPreThreads, kPreThreads == 256 ? 3 : 6) preprocess_kernel(PreprocessArgs a) {
  chain_wait();
  chain_release();
  constexpr int nk = (kDeg + 1) * (kDeg + 1);
  constexpr int kPlanes = kGeomPlanes + 3 * nk;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  PreprocessSmem<kDeg>& sm = *reinterpret_cast<PreprocessSmem<kDeg>*>(smem_raw);
  const int tid = threadIdx.x;
  // Slices are taken from the last to the first: the fused backward + Adam pass
  // of the previous step walks the parameters upwards, so the last slices'
  // parameters are still in L2 when this kernel starts.
  const int64_t blk = static_cast<int64_t>(gridDim.x) - 1 - static_cast<int64_t>(blockIdx.x);
  const int64_t i0 = blk * kPreThreads;
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
    // The CTA that will start about when this one ends (one grid of resident
    // CTAs later) finds its planes in L2: its copies then wait on L2, not on
    // DRAM, and this CTA's copies overlap the DRAM reads of the next slices.
    const int64_t nb = blk - a.prefetch_ahead;
    if (a.prefetch_ahead > 0 && nb >= 0) {
      const int64_t j0 = nb * kPreThreads;
      const uint32_t pbytes = static_cast<uint32_t>(np - j0 < kPreThreads ? np - j0 : kPreThreads) * 4u;
#pragma unroll
      for (int c = 0; c < 3; ++c) bulk_prefetch_l2(a.means + c * np + j0, pbytes);
#pragma unroll
      for (int c = 0; c < 3; ++c) bulk_prefetch_l2(a.log_scales + c * np + j0, pbytes);
#pragma unroll
      for (int c = 0; c < 4; ++c) bulk_prefetch_l2(a.quats + c * np + j0, pbytes);
      bulk_prefetch_l2(a.opacity_logits + j0, pbytes);
      for (int ch = 0; ch < 3; ++ch)
        for (int k = 0; k < nk; ++k)
          bulk_prefetch_l2(a.sh + (static_cast<int64_t>(ch) * a.sh_k + k) * np + j0, pbytes);
    }
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
    if (tid == 0) a.block_sums[blk] = make_uint2(0u, 0u);
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
      const float q4[4] = {sm.plane[6][tid], sm.plane[7][tid], sm.plane[8][tid], sm.plane[9][tid]};
      const float ls3[3] = {sm.plane[3][tid], sm.plane[4][tid], sm.plane[5][tid]};
      const double iz = 1.0 / Z;
      const double u = cam.fx * X * iz + cam.cx;
      const double v = cam.fy * Y * iz + cam.cy;
      const float sig = 1.0f / (1.0f + expf(-sm.plane[10][tid]));
      // The covariance chain in float32. The tile rect is an integer decision:
      // where a rect bound lies within 1e-4 r + 1e-3 px of a tile boundary (far
      // beyond the float32 error of r) the chain is redone in float64, the
      // precision in which the rect is defined, so rects never depend on the
      // float32 rounding.
      const ScreenCov<float> vf = screen_cov<float>(q4, ls3, X, Y, Z, cam);
      float comp = compensation<float>(vf, a.mip_comp != 0);
      double rad = rect_radius<float>(vf, a.opacity_rect != 0, sig * comp);
      float ca = vf.a0 + static_cast<float>(kDilation), cc = vf.c0 + static_cast<float>(kDilation), cb = vf.b0;
      float det = vf.det0 + static_cast<float>(kDilation) * (vf.a0 + vf.c0) +
                  static_cast<float>(kDilation * kDilation);
      {
        const double m = (1e-4 * rad + 1e-3) / kTile;
        const bool sure = clear_of_integers((u - rad - (kTile - 1)) / kTile, m) &&
                          clear_of_integers((u + rad) / kTile, m) &&
                          clear_of_integers((v - rad - (kTile - 1)) / kTile, m) &&
                          clear_of_integers((v + rad) / kTile, m) && rad == rad;
        if (!sure) {
          const ScreenCov<double> vd = screen_cov<double>(q4, ls3, X, Y, Z, cam);
          const double compd = compensation<double>(vd, a.mip_comp != 0);
          rad = rect_radius<double>(vd, a.opacity_rect != 0, static_cast<double>(sig) * compd);
          comp = static_cast<float>(compd);
          ca = static_cast<float>(vd.a0 + kDilation);
          cc = static_cast<float>(vd.c0 + kDilation);
          cb = static_cast<float>(vd.b0);
          det = static_cast<float>(vd.det0 + kDilation * (vd.a0 + vd.c0) + kDilation * kDilation);
        }
      }
      if (det > 0.0f) {
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
          const float opacity = sig * comp;
          // view-dependent colour at v = normalize(p - campos); its SH planes
          // were still arriving while the geometry above ran
          sh_ok = mbar_wait(&sm.bar[1], 0, 1 << 16);
          const float d[3] = {static_cast<float>(p[0] - cam.campos[0]), static_cast<float>(p[1] - cam.campos[1]),
                              static_cast<float>(p[2] - cam.campos[2])};
          const float idn = rsqrtf(d[0] * d[0] + d[1] * d[1] + d[2] * d[2]);
          float Yk[16];
          sh_basis(kDeg, d[0] * idn, d[1] * idn, d[2] * idn, Yk);
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
          const float E = logf(255.0f * opacity);
          float hx = -1.0f, hy = -1.0f;
          if (E > 0.0f) {
            hx = sqrtf(2.0f * E * ca) * 1.001f + 0.02f;
            hy = sqrtf(2.0f * E * cc) * 1.001f + 0.02f;
          }
          const float idet = kLog2e / det;
          s.a = make_float4(static_cast<float>(u), static_cast<float>(v), hx, hy);
          s.b = make_float4(-0.5f * cc * idet, cb * idet, -0.5f * ca * idet, log2f(opacity));
          s.c = make_float4(rgb[0], rgb[1], rgb[2], opacity);
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
  __shared__ uint32_t s_sum[kPreThreads / 32];
  __shared__ uint32_t s_vis[kPreThreads / 32];
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
    a.block_sums[blk] = make_uint2(b, v);
  }
}

// Exclusive prefix of the per-block visible counts (one CTA of 1024 threads),
// plus the entry and visible totals and the depth-key range copied into the
// readback record.
__global__ void __launch_bounds__(1024) scan_blocks_kernel(const uint2* block_sums, int64_t nb,
                                                           uint32_t* visible_prefix,
                                                           const uint32_t* depth_range,
                                                           ForwardInfo* info) {
  chain_wait();
  chain_release();
  __shared__ uint64_t s_warp[32];
  __shared__ uint32_t s_vwarp[32];
  const int tid = threadIdx.x;
  const int64_t per = (nb + blockDim.x - 1) / blockDim.x;
  const int64_t lo = tid * per, hi = min(nb, lo + per);
  // each thread's run is read kRun sums at a time, all loads of a group in
  // flight together (a thread has about a dozen sums at 3M Gaussians)
  constexpr int kRun = 8;
  uint64_t entries = 0;
  uint32_t local = 0;
  for (int64_t k0 = lo; k0 < hi; k0 += kRun) {
    uint2 b[kRun];
#pragma unroll
    for (int u = 0; u < kRun; ++u) b[u] = k0 + u < hi ? block_sums[k0 + u] : make_uint2(0u, 0u);
#pragma unroll
    for (int u = 0; u < kRun; ++u) {
      entries += b[u].x;
      local += b[u].y;
    }
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
  for (int64_t k0 = lo; k0 < hi; k0 += kRun) {
    uint32_t c[kRun];
#pragma unroll
    for (int u = 0; u < kRun; ++u) c[u] = k0 + u < hi ? block_sums[k0 + u].y : 0u;
#pragma unroll
    for (int u = 0; u < kRun; ++u) {
      if (k0 + u < hi) visible_prefix[k0 + u] = run;
      run += c[u];
    }
  }
  if (tid == 0) {
    info->num_entries = s_warp[0];
    info->num_visible = s_vwarp[31];
    info->depth_min = depth_range[0];
    info->depth_max = depth_range[1];
  }
}

template <int kDeg>
cudaError_t launch_preprocess_deg(const PreprocessArgs& args, unsigned grid, cudaStream_t st) {
  const int smem = static_cast<int>(sizeof(PreprocessSmem<kDeg>));
  cudaError_t e = cudaFuncSetAttribute(preprocess_kernel<kDeg>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // resident CTAs: SMs x CTAs per SM
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, preprocess_kernel<kDeg>, kPreThreads, smem);
  if (e != cudaSuccess) return e;
  PreprocessArgs a = args;
  a.prefetch_ahead = static_cast<int64_t>(sms) * per_sm;
  return launch_chained(preprocess_kernel<kDeg>, dim3(grid), dim3(kPreThreads), smem, st, a);
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
  return launch_chained(scan_blocks_kernel, dim3(1), dim3(1024), 0, st, block_sums, num_blocks, visible_prefix,
                        depth_range, info);
}

}  // namespace gs
