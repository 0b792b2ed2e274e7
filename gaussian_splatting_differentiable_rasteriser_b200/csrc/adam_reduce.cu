// Data-parallel exchange fused with Adam: one kernel reads every rank's
// gradient for this rank's shard (peer memory over NVLink / NVSwitch, or local
// memory), averages them in a fixed rank order, applies the Adam step to the
// shard and stores the updated parameters into every other rank's parameter
// buffer. It replaces reduce-scatter -> Adam -> all-gather (three launches,
// two of them collectives) with one pass whose NVLink traffic is the same as
// the two collectives' (each remote gradient read once, each updated
// parameter written once per peer) and whose HBM traffic is one Adam step's.
//
// Method: "How a computer rebuilds a real place ... Gaussian Splats"
// (taosengine.com), section "Per step" (one photo per step; with one photo per
// rank the batch gradient is the mean of the ranks' gradients) and the Adam
// paragraph after "Proving the blame is right".
//
// B200 design: HBM / NVLink bound. float4 accesses when every pointer is 16-byte
// aligned, a grid of 148 x 8 CTAs striding over the shard, the per-rank
// gradient loads of one item issued together so the NVLink latency overlaps,
// plain (non-multicast) loads and stores only. The kernel never waits on
// another GPU: the caller orders it after every rank's backward and before any
// rank's next forward with stream-ordered barriers.
#include "adam_math.cuh"
#include "gs_kernels.cuh"

namespace gs {

namespace {

constexpr int kReduceThreads = 256;

__device__ __forceinline__ float4 ld4(const float* p, int64_t i) {
  return __ldcg(reinterpret_cast<const float4*>(p) + i);
}

// R = the number of gradient sources (ranks), a template argument so the loads
// of one item are all in flight at once and no register holds an unused rank
template <int R>
__global__ void __launch_bounds__(kReduceThreads) adam_reduce_vec_kernel(ReduceAdamArgs a) {
  const int64_t n4 = a.count >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kReduceThreads;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kReduceThreads + threadIdx.x; i < n4; i += stride) {
    float4 gr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) gr[r] = ld4(a.grads[r], i);
    // fixed rank order: the same sum on every GPU and in every run
    float4 g = gr[0];
#pragma unroll
    for (int r = 1; r < R; ++r) {
      g.x += gr[r].x;
      g.y += gr[r].y;
      g.z += gr[r].z;
      g.w += gr[r].w;
    }
    g.x *= a.grad_scale;
    g.y *= a.grad_scale;
    g.z *= a.grad_scale;
    g.w *= a.grad_scale;
    float4 p = reinterpret_cast<float4*>(a.p)[i];
    float4 m = reinterpret_cast<float4*>(a.m)[i];
    float4 v = reinterpret_cast<float4*>(a.v)[i];
    adam_one(p.x, g.x, m.x, v.x, a.s);
    adam_one(p.y, g.y, m.y, v.y, a.s);
    adam_one(p.z, g.z, m.z, v.z, a.s);
    adam_one(p.w, g.w, m.w, v.w, a.s);
    reinterpret_cast<float4*>(a.p)[i] = p;
    reinterpret_cast<float4*>(a.m)[i] = m;
    reinterpret_cast<float4*>(a.v)[i] = v;
#pragma unroll
    for (int d = 0; d < kMaxRanks; ++d)
      if (d < a.n_copies) __stcg(reinterpret_cast<float4*>(a.copies[d]) + i, p);
    if (a.zero_grads) {
#pragma unroll
      for (int r = 0; r < R; ++r) reinterpret_cast<float4*>(a.grads[r])[i] = zero;
    }
  }
  // make the peer stores visible system-wide before the kernel is seen as done
  if (a.n_copies > 0 || (a.zero_grads && R > 1)) __threadfence_system();
}

template <int R>
__global__ void __launch_bounds__(kReduceThreads) adam_reduce_scalar_kernel(ReduceAdamArgs a) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kReduceThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kReduceThreads + threadIdx.x; i < a.count;
       i += stride) {
    float gr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) gr[r] = __ldcg(a.grads[r] + i);
    float g = gr[0];
#pragma unroll
    for (int r = 1; r < R; ++r) g += gr[r];
    g *= a.grad_scale;
    float p = a.p[i], m = a.m[i], v = a.v[i];
    adam_one(p, g, m, v, a.s);
    a.p[i] = p;
    a.m[i] = m;
    a.v[i] = v;
#pragma unroll
    for (int d = 0; d < kMaxRanks; ++d)
      if (d < a.n_copies) __stcg(a.copies[d] + i, p);
    if (a.zero_grads) {
#pragma unroll
      for (int r = 0; r < R; ++r) a.grads[r][i] = 0.0f;
    }
  }
  if (a.n_copies > 0 || (a.zero_grads && R > 1)) __threadfence_system();
}

bool all_aligned16(const ReduceAdamArgs& a) {
  uintptr_t bits = reinterpret_cast<uintptr_t>(a.p) | reinterpret_cast<uintptr_t>(a.m) |
                   reinterpret_cast<uintptr_t>(a.v);
  for (int r = 0; r < a.n_grads; ++r) bits |= reinterpret_cast<uintptr_t>(a.grads[r]);
  for (int d = 0; d < a.n_copies; ++d) bits |= reinterpret_cast<uintptr_t>(a.copies[d]);
  return (bits & 15u) == 0;
}

unsigned grid_for(int64_t items) {
  const int64_t want = (items + kReduceThreads - 1) / kReduceThreads;
  return static_cast<unsigned>(want < 148 * 8 ? (want > 0 ? want : 1) : 148 * 8);
}

template <int R>
cudaError_t launch_ranks(const ReduceAdamArgs& a, cudaStream_t st) {
  if (all_aligned16(a) && (a.count & 3) == 0) {
    adam_reduce_vec_kernel<R><<<grid_for(a.count >> 2), kReduceThreads, 0, st>>>(a);
  } else {
    adam_reduce_scalar_kernel<R><<<grid_for(a.count), kReduceThreads, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_adam_reduce(const ReduceAdamArgs& a, cudaStream_t st) {
  if (a.count == 0) return cudaSuccess;
  static_assert(kMaxRanks == 8, "one instantiation per rank count");
  switch (a.n_grads) {
    case 1: return launch_ranks<1>(a, st);
    case 2: return launch_ranks<2>(a, st);
    case 3: return launch_ranks<3>(a, st);
    case 4: return launch_ranks<4>(a, st);
    case 5: return launch_ranks<5>(a, st);
    case 6: return launch_ranks<6>(a, st);
    case 7: return launch_ranks<7>(a, st);
    case 8: return launch_ranks<8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gs
