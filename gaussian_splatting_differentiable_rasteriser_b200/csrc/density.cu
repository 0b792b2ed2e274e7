// Adaptive density control between training steps: prune / clone / split
// with stream compaction, and the opacity reset.
//
// Method: "Gaussian splatting training" study notes (bailiping.com), slides
// "Where to add capacity" and "A separate heuristic" (average screen-space
// centre gradient over the views that saw a Gaussian; small flagged Gaussians
// cloned, large ones split into two children sampled around the parent with
// smaller scales; very low opacity pruned; reset clamps opacity to at most
// 0.01); "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), section "Densification" (halves shrink by 1.6, reshaped
// Gaussians restart their Adam moments).
//
// B200 design: two passes over the Gaussians plus a one-CTA scan. The first
// classifies every Gaussian and reduces per-256-block counts of kept Gaussians,
// clones and splits; the scan turns them into block offsets and totals (read
// back once, for the capacity check); the second pass classifies again, ranks
// each Gaussian inside its block with warp ballots, and writes its output
// columns: kept Gaussians (parents of clones included) first in index order,
// then the clones, then the split children, so kept runs stay contiguous and
// the planar writes coalesce. Every decision is taken in float64 against
// thresholds converted once on the host, so it is exact.
#include "gs_kernels.cuh"

namespace gs {

namespace {

enum Category : int { kPruned = 0, kKept = 1, kCloned = 2, kSplit = 3 };

__device__ __forceinline__ int classify(const DensifyArgs& a, int64_t i) {
  const int64_t np = a.np_in;
  if (static_cast<double>(a.opacity_logits[i]) < a.logit_threshold) return kPruned;
  const uint32_t cnt = a.view_count[i];
  const bool dense = cnt > 0u && static_cast<double>(a.grad_accum[i]) / static_cast<double>(cnt) >=
                                     a.grad_threshold;
  if (!dense) return kKept;
  const float ls_max = fmaxf(fmaxf(a.log_scales[i], a.log_scales[np + i]), a.log_scales[2 * np + i]);
  return static_cast<double>(ls_max) > a.log_scale_threshold ? kSplit : kCloned;
}

// Block-exclusive ranks of three flags over the block's threads in index
// order, and the block totals (written by thread 0 when `totals_out`).
struct Ranks {
  uint32_t kept, clone, split;
};

__device__ __forceinline__ Ranks block_ranks(bool kept, bool clone, bool split, uint4* totals_out) {
  __shared__ uint32_t s_w[3][kDensifyBlock / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned mk = __ballot_sync(0xffffffffu, kept);
  const unsigned mc = __ballot_sync(0xffffffffu, clone);
  const unsigned ms = __ballot_sync(0xffffffffu, split);
  if (lane == 0) {
    s_w[0][warp] = __popc(mk);
    s_w[1][warp] = __popc(mc);
    s_w[2][warp] = __popc(ms);
  }
  __syncthreads();
  Ranks r{static_cast<uint32_t>(__popc(mk & lt)), static_cast<uint32_t>(__popc(mc & lt)),
          static_cast<uint32_t>(__popc(ms & lt))};
  uint32_t tk = 0, tc = 0, ts = 0;
  for (int k = 0; k < kDensifyBlock / 32; ++k) {
    if (k < warp) {
      r.kept += s_w[0][k];
      r.clone += s_w[1][k];
      r.split += s_w[2][k];
    }
    tk += s_w[0][k];
    tc += s_w[1][k];
    ts += s_w[2][k];
  }
  if (totals_out && threadIdx.x == 0) *totals_out = make_uint4(tk, tc, ts, 0u);
  return r;
}

__global__ void __launch_bounds__(kDensifyBlock) densify_count_kernel(DensifyArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kDensifyBlock + threadIdx.x;
  const int cat = i < a.n ? classify(a, i) : kPruned;
  block_ranks(cat == kKept || cat == kCloned, cat == kCloned, cat == kSplit, a.block_counts + blockIdx.x);
}

// Exclusive prefixes of the per-block counts (one CTA) and the totals.
__global__ void __launch_bounds__(1024) densify_scan_kernel(const uint4* counts, int64_t nb, uint4* prefix,
                                                            uint4* totals) {
  __shared__ uint4 s_w[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t per = (nb + blockDim.x - 1) / blockDim.x;
  const int64_t lo = tid * per, hi = min(nb, lo + per);
  uint4 loc = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t k = lo; k < hi; ++k) {
    const uint4 c = counts[k];
    loc.x += c.x;
    loc.y += c.y;
    loc.z += c.z;
  }
  uint4 v = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t nx = __shfl_up_sync(0xffffffffu, v.x, o), ny = __shfl_up_sync(0xffffffffu, v.y, o),
                   nz = __shfl_up_sync(0xffffffffu, v.z, o);
    if (lane >= o) {
      v.x += nx;
      v.y += ny;
      v.z += nz;
    }
  }
  if (lane == 31) s_w[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint4 w = s_w[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t nx = __shfl_up_sync(0xffffffffu, w.x, o), ny = __shfl_up_sync(0xffffffffu, w.y, o),
                     nz = __shfl_up_sync(0xffffffffu, w.z, o);
      if (lane >= o) {
        w.x += nx;
        w.y += ny;
        w.z += nz;
      }
    }
    s_w[lane] = w;
  }
  __syncthreads();
  uint4 run = make_uint4(v.x - loc.x, v.y - loc.y, v.z - loc.z, 0u);
  if (warp > 0) {
    run.x += s_w[warp - 1].x;
    run.y += s_w[warp - 1].y;
    run.z += s_w[warp - 1].z;
  }
  for (int64_t k = lo; k < hi; ++k) {
    prefix[k] = run;
    const uint4 c = counts[k];
    run.x += c.x;
    run.y += c.y;
    run.z += c.z;
  }
  if (tid == 0) *totals = make_uint4(s_w[31].x, s_w[31].y, s_w[31].z, 0u);
}

// Writes Gaussian i's parameters into output column d (planar, stride np_out),
// with the log-scales and means optionally replaced; moments copied or zeroed.
__device__ __forceinline__ void write_column(const DensifyArgs& a, int64_t i, int64_t d, bool keep_moments,
                                             const float* means, const float* log_scales) {
  const int64_t ni = a.np_in, no = a.np_out;
  const float* src[5] = {a.means, a.log_scales, a.quats, a.opacity_logits, a.sh};
  const int planes[5] = {3, 3, 4, 1, 3 * a.sh_k};
#pragma unroll
  for (int g = 0; g < 5; ++g) {
    for (int c = 0; c < planes[g]; ++c) {
      float val = src[g][c * ni + i];
      if (g == 0 && means) val = means[c];
      if (g == 1 && log_scales) val = log_scales[c];
      a.out_p[g][c * no + d] = val;
      a.out_m[g][c * no + d] = keep_moments ? a.m[g][c * ni + i] : 0.0f;
      a.out_v[g][c * no + d] = keep_moments ? a.v[g][c * ni + i] : 0.0f;
    }
  }
}

__global__ void __launch_bounds__(kDensifyBlock) densify_write_kernel(DensifyArgs a, uint4 tot) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kDensifyBlock + threadIdx.x;
  const int cat = i < a.n ? classify(a, i) : kPruned;
  const Ranks r = block_ranks(cat == kKept || cat == kCloned, cat == kCloned, cat == kSplit, nullptr);
  if (cat == kPruned) return;
  const uint4 P = a.block_prefix[blockIdx.x];
  if (cat == kKept || cat == kCloned) write_column(a, i, P.x + r.kept, true, nullptr, nullptr);
  if (cat == kCloned) write_column(a, i, static_cast<int64_t>(tot.x) + P.y + r.clone, false, nullptr, nullptr);
  if (cat == kSplit) {
    const int64_t np = a.np_in;
    // children at mean + R(q/|q|) diag(exp(log-scales)) z_k, log-scales - ln 1.6
    const double qw = a.quats[i], qx = a.quats[np + i], qy = a.quats[2 * np + i], qz = a.quats[3 * np + i];
    const double qn = sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
    const double w = qw / qn, x = qx / qn, y = qy / qn, z = qz / qn;
    const double R[9] = {1.0 - 2.0 * (y * y + z * z), 2.0 * (x * y - w * z), 2.0 * (x * z + w * y),
                         2.0 * (x * y + w * z), 1.0 - 2.0 * (x * x + z * z), 2.0 * (y * z - w * x),
                         2.0 * (x * z - w * y), 2.0 * (y * z + w * x), 1.0 - 2.0 * (x * x + y * y)};
    double ls[3], s[3];
    float ls_child[3];
    for (int c = 0; c < 3; ++c) {
      ls[c] = a.log_scales[c * np + i];
      s[c] = exp(ls[c]);
      ls_child[c] = static_cast<float>(ls[c] - log(1.6));
    }
    const int64_t first = static_cast<int64_t>(tot.x) + tot.y + 2 * (static_cast<int64_t>(P.z) + r.split);
    for (int k = 0; k < 2; ++k) {
      const float* zk = a.normals + (i * 2 + k) * 3;
      const double sz[3] = {s[0] * zk[0], s[1] * zk[1], s[2] * zk[2]};
      float mean[3];
      for (int c = 0; c < 3; ++c)
        mean[c] = static_cast<float>(static_cast<double>(a.means[c * np + i]) + R[3 * c] * sz[0] +
                                     R[3 * c + 1] * sz[1] + R[3 * c + 2] * sz[2]);
      write_column(a, i, first + k, false, mean, ls_child);
    }
  }
}

// ------------------------------------------------------------- relocation
// "How a computer rebuilds a real place ... Gaussian Splats", section
// "Densification: cloning the busy blobs, recycling the dead": dead Gaussians
// (opacity < ~0.02) are moved next to donors (opacity > ~0.4), the largest
// donors first; both halves shrink by 1.6 and restart their Adam moments.
// Classification, compaction (dead indices; donors with a descending-size key)
// and, after a stable sort of the donors, one thread per pair.

enum RelocClass : int { kRelocNone = 0, kRelocDead = 1, kRelocDonor = 2 };

__device__ __forceinline__ int reloc_class(const RelocateArgs& a, int64_t i) {
  const double logit = a.p[3][i];
  if (logit < a.dead_logit) return kRelocDead;
  if (logit > a.donor_logit) return kRelocDonor;
  return kRelocNone;
}

// Largest log-scale as a key that sorts ascending for descending size (the
// float's bits mapped to an order-preserving unsigned integer, then inverted).
__device__ __forceinline__ uint32_t size_key(const RelocateArgs& a, int64_t i) {
  const float* ls = a.p[1];
  const float s = fmaxf(fmaxf(ls[i], ls[a.np + i]), ls[2 * a.np + i]);
  const uint32_t u = __float_as_uint(s);
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~ord;
}

__global__ void __launch_bounds__(kDensifyBlock) relocate_count_kernel(RelocateArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kDensifyBlock + threadIdx.x;
  const int c = i < a.n ? reloc_class(a, i) : kRelocNone;
  block_ranks(c == kRelocDead, c == kRelocDonor, false, a.block_counts + blockIdx.x);
}

__global__ void __launch_bounds__(kDensifyBlock) relocate_compact_kernel(RelocateArgs a) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kDensifyBlock + threadIdx.x;
  const int c = i < a.n ? reloc_class(a, i) : kRelocNone;
  const Ranks r = block_ranks(c == kRelocDead, c == kRelocDonor, false, nullptr);
  const uint4 P = a.block_prefix[blockIdx.x];
  if (c == kRelocDead) {
    const int64_t k = static_cast<int64_t>(P.x) + r.kept;
    if (k < a.n) a.dead[k] = static_cast<uint32_t>(i);
    else record_error(a.err, kErrIndexRange);
  } else if (c == kRelocDonor) {
    const int64_t k = static_cast<int64_t>(P.y) + r.clone;
    if (k < a.n) {
      a.donor_keys[k] = size_key(a, i);
      a.donor_vals[k] = static_cast<uint32_t>(i);
    } else {
      record_error(a.err, kErrIndexRange);
    }
  }
}

__global__ void relocate_pair_kernel(RelocateArgs a) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= a.pairs) return;
  const int64_t d = a.dead[j], b = a.sorted_donors[j];
  const int64_t np = a.np;
  if (d >= a.n || b >= a.n) {
    record_error(a.err, kErrIndexRange);
    return;
  }
  // the donor's own Gaussian: mean + R(q/|q|) diag(exp(log-scales)) z_j
  const float* q = a.p[2];
  const double qw = q[b], qx = q[np + b], qy = q[2 * np + b], qz = q[3 * np + b];
  const double qn = sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
  const double w = qw / qn, x = qx / qn, y = qy / qn, z = qz / qn;
  const double R[9] = {1.0 - 2.0 * (y * y + z * z), 2.0 * (x * y - w * z), 2.0 * (x * z + w * y),
                       2.0 * (x * y + w * z), 1.0 - 2.0 * (x * x + z * z), 2.0 * (y * z - w * x),
                       2.0 * (x * z - w * y), 2.0 * (y * z + w * x), 1.0 - 2.0 * (x * x + y * y)};
  const float* zj = a.normals + 3 * j;
  double sz[3];
  float ls_new[3], mean[3];
  for (int c = 0; c < 3; ++c) {
    const double ls = a.p[1][c * np + b];
    sz[c] = exp(ls) * zj[c];
    ls_new[c] = static_cast<float>(ls - log(1.6));
  }
  for (int c = 0; c < 3; ++c)
    mean[c] = static_cast<float>(static_cast<double>(a.p[0][c * np + b]) + R[3 * c] * sz[0] + R[3 * c + 1] * sz[1] +
                                 R[3 * c + 2] * sz[2]);
  const int planes[5] = {3, 3, 4, 1, 3 * a.sh_k};
  for (int g = 0; g < 5; ++g)
    for (int c = 0; c < planes[g]; ++c) {
      const int64_t o = c * np;
      a.p[g][o + d] = a.p[g][o + b];
      a.m[g][o + d] = 0.0f;
      a.v[g][o + d] = 0.0f;
      a.m[g][o + b] = 0.0f;
      a.v[g][o + b] = 0.0f;
    }
  for (int c = 0; c < 3; ++c) {
    a.p[0][c * np + d] = mean[c];
    a.p[1][c * np + d] = ls_new[c];
    a.p[1][c * np + b] = ls_new[c];
  }
}

__global__ void opacity_reset_kernel(float* logits, float* m, float* v, int64_t n, float cap) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  logits[i] = fminf(logits[i], cap);
  m[i] = 0.0f;
  v[i] = 0.0f;
}

}  // namespace

cudaError_t launch_densify_count(const DensifyArgs& a, cudaStream_t st) {
  const int64_t nb = (a.n + kDensifyBlock - 1) / kDensifyBlock;
  if (nb > 0) densify_count_kernel<<<static_cast<unsigned>(nb), kDensifyBlock, 0, st>>>(a);
  densify_scan_kernel<<<1, 1024, 0, st>>>(a.block_counts, nb, a.block_prefix, a.totals);
  return cudaGetLastError();
}

cudaError_t launch_densify_write(const DensifyArgs& a, uint4 totals, cudaStream_t st) {
  const int64_t nb = (a.n + kDensifyBlock - 1) / kDensifyBlock;
  if (nb == 0) return cudaSuccess;
  densify_write_kernel<<<static_cast<unsigned>(nb), kDensifyBlock, 0, st>>>(a, totals);
  return cudaGetLastError();
}

cudaError_t launch_relocate_classify(const RelocateArgs& a, cudaStream_t st) {
  const int64_t nb = (a.n + kDensifyBlock - 1) / kDensifyBlock;
  if (nb > 0) relocate_count_kernel<<<static_cast<unsigned>(nb), kDensifyBlock, 0, st>>>(a);
  densify_scan_kernel<<<1, 1024, 0, st>>>(a.block_counts, nb, a.block_prefix, a.totals);
  if (nb > 0) relocate_compact_kernel<<<static_cast<unsigned>(nb), kDensifyBlock, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_relocate_pairs(const RelocateArgs& a, cudaStream_t st) {
  if (a.pairs == 0) return cudaSuccess;
  relocate_pair_kernel<<<static_cast<unsigned>((a.pairs + 127) / 128), 128, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_opacity_reset(float* logits, float* m, float* v, int64_t n, float cap, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  opacity_reset_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(logits, m, v, n, cap);
  return cudaGetLastError();
}

}  // namespace gs
