// Kernel argument records and host-side launchers of the rasteriser stages.
// Everything here is internal to the library; the public surface is gs_api.h.
#pragma once

#include "adam_math.cuh"
#include "gs_common.cuh"

namespace gs {

// Programmatic dependent launch. The kernels of a training step are launched
// with launch_chained: a kernel's CTAs may then be scheduled while the kernel
// before it on the stream is still finishing, so that the launch of each stage
// overlaps the tail of the previous one. Every such kernel calls chain_wait()
// first, before it reads or writes anything (it returns once the previous
// kernel has completed and its writes are visible; a no-op for a kernel
// launched the ordinary way), and then chain_release(), which lets the next
// kernel be scheduled once all of this kernel's CTAs have started.
__device__ __forceinline__ void chain_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void chain_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... P, typename... A>
inline cudaError_t launch_chained(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  A&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<A&&>(args)...);
}

// Written by the preprocess + block scan and read back by the host before the
// sort: the entry count, the number of visible Gaussians and the range of
// depth keys of visible Gaussians.
struct ForwardInfo {
  uint64_t num_entries;
  uint32_t num_visible;
  uint32_t depth_min, depth_max;
  uint32_t device_error;
};

// Gaussians per preprocess CTA, and the granularity of the per-block totals
// (tiles touched, visible Gaussians) that the block scan and the compaction use.
#ifndef GS_PRE_BLOCK
#define GS_PRE_BLOCK 256
#endif
constexpr int kGaussBlock = GS_PRE_BLOCK;
static_assert(kGaussBlock == 128 || kGaussBlock == 256, "preprocess block");

struct PreprocessArgs {
  const float *means, *log_scales, *quats, *opacity_logits, *sh;
  int64_t n, n_pad;
  int sh_k;           // coefficients stored per channel, (sh_degree + 1)^2
  int active_degree;  // bands used
  CamArgs cam;
  Screen* screen;
  float* depth;
  uint2* rect;  // x0 | x1 << 16, y0 | y1 << 16 (inclusive tile indices)
  uint32_t* touched;
  uint8_t* clamped;
  uint2* block_sums;      // per 256-Gaussian block: (tiles touched, visible Gaussians)
  uint32_t* depth_range;  // [min, max] of visible depth keys (atomics)
  uint32_t* err;          // device error word
  int opacity_rect;       // opacity-aware tile rect (GS_OPTION_OPACITY_RECT)
  int mip_comp;           // opacity times the compensation factor (GS_OPTION_MIP_COMPENSATION)
  int64_t prefetch_ahead; // set by the launcher: CTA b prefetches slice b + this into L2
};

cudaError_t launch_preprocess(const PreprocessArgs& a, int64_t num_blocks, cudaStream_t st);
// Exclusive prefix of the per-block visible counts, plus the totals and the
// depth-key range copied into the readback record.
cudaError_t launch_scan_blocks(const uint2* block_sums, int64_t num_blocks, uint32_t* visible_prefix,
                               const uint32_t* depth_range, ForwardInfo* info, cudaStream_t st);

// ---------------------------------------------------------------- sorting
// Stable LSD radix sort of 32-bit keys with 32-bit values.
struct SortPlan {
  int64_t n;      // items
  int key_bits;   // significant low bits of the keys
  int passes;     // ceil(key_bits / 8)
  int64_t tiles;  // chunks of kSortTileKeys keys (one CTA each)
};

// Radix-pass shape: threads per CTA (a multiple of 256), keys per thread and
// the minimum CTAs per SM the downsweep is compiled for (build-time tunables;
// 512 x 8 at two CTAs per SM measured fastest on B200: the pass is bound by
// the latency of its ranking chain, so resident warps matter most).
#ifndef GS_SORT_THREADS
#define GS_SORT_THREADS 512
#endif
#ifndef GS_SORT_ITEMS
#define GS_SORT_ITEMS 8
#endif
#ifndef GS_SORT_MINB
#define GS_SORT_MINB 2
#endif
constexpr int kSortThreads = GS_SORT_THREADS;
constexpr int kSortItems = GS_SORT_ITEMS;
constexpr int kSortTileKeys = kSortThreads * kSortItems;
static_assert(kSortThreads % 256 == 0 && kSortItems % 4 == 0, "radix-pass shape");
constexpr int kRadix = 256;
constexpr int kMaxPasses = 4;

// Visible Gaussians in index order as (depth key - depth_min, index).
struct CompactArgs {
  int64_t n;
  const uint32_t* touched;
  const float* depth;
  const uint32_t* visible_prefix;  // per 256-Gaussian block
  uint32_t depth_min;
  int64_t max_out;
  uint32_t* keys;
  uint32_t* vals;
  uint32_t* err;
};
cudaError_t launch_compact(const CompactArgs& a, int64_t num_blocks, cudaStream_t st);

// One (tile, index) entry per tile touched by each visible Gaussian, in the
// depth order given by `order`: the tiles touched by each chunk of kDupItems
// Gaussians are counted, scanned, and each chunk's CTA writes its entries from
// its offset (no wait between CTAs).
struct DuplicateArgs {
  int64_t count;          // visible Gaussians
  const uint32_t* order;  // Gaussian indices sorted by depth
  const uint32_t* touched;
  const uint2* rect;
  int tiles_x;
  int64_t max_entries;
  uint32_t* keys;           // tile
  uint32_t* vals;           // Gaussian index
  uint32_t* chunk_offsets;  // [ceil(count / kDupItems)] scratch: tiles per chunk, then their prefix
  uint32_t* err;
};
#ifndef GS_DUP_PER_THREAD
#define GS_DUP_PER_THREAD 2
#endif
constexpr int kDupThreads = 256;
constexpr int kDupPerThread = GS_DUP_PER_THREAD;  // visible Gaussians per thread of a duplicate CTA
constexpr int kDupItems = kDupThreads * kDupPerThread;
cudaError_t launch_duplicate(const DuplicateArgs& a, cudaStream_t st);

struct SortBuffers {
  uint32_t* keys[2];
  uint32_t* vals[2];
  uint32_t* hist;      // [kMaxPasses][256] digit counts
  uint32_t* offsets;   // [kMaxPasses][256] exclusive digit offsets
  uint32_t* chunk_counts;  // [kMaxPasses][256][tiles] per-chunk digit counts, then their offsets
  uint32_t* err;
};

// Sorts keys[0]/vals[0]; returns in *out_buf the buffer (0 or 1) holding the result.
cudaError_t launch_sort(const SortPlan& plan, const SortBuffers& b, int* out_buf, cudaStream_t st);

// Per-tile [first, last) of the tile-sorted entries (keys = tile indices).
cudaError_t launch_ranges(const uint32_t* keys, int64_t n, uint2* ranges, int64_t num_tiles,
                          cudaStream_t st);
// The tiles in descending order of list length (by powers of two), the order
// in which the blend kernels take them.
cudaError_t launch_tile_order(const uint2* ranges, int64_t num_tiles, uint32_t* order, cudaStream_t st);

// ---------------------------------------------------------------- blending
struct BlendArgs {
  const uint2* ranges;
  const uint32_t* tile_order;  // CTA b blends tile tile_order[b]
  const uint32_t* order;  // sorted Gaussian index per entry
  const Screen* screen;
  CamArgs cam;
  // forward outputs / backward inputs
  float* image;
  float* final_T;
  int32_t* n_contrib;
  // backward only
  const float* dimage;
  float* sgrad;  // [n][kGradStride]
  // when not null: pairs[0] += (pixel, Gaussian) pairs the method's walk visits,
  // pairs[2] += pairs that blend (alpha >= 1/255 before the walk stops)
  unsigned long long* pairs;
  // per warp (8 per tile) the entries that pass its box test and blend at one
  // of its pixels, written by the forward and walked by the backward: (list
  // position, Gaussian) in list order, warp w of a tile with list [beg, end) at
  // surv[8 beg + w (end - beg)]
  uint2* surv;
  uint32_t* surv_count;  // [tiles][8]
  // backward in deterministic mode: the raw sums in fixed point ([n][9], zeroed)
  unsigned long long* sgrad_fixed;
};

cudaError_t launch_blend_forward(const BlendArgs& a, cudaStream_t st);
cudaError_t launch_blend_backward(const BlendArgs& a, cudaStream_t st);
cudaError_t launch_decode_fixed(const unsigned long long* fixed, int64_t n, float* sgrad, cudaStream_t st);

// ---------------------------------------------------------------- loss
struct LossArgs {
  const float* x;
  const float* y;
  int height, width;
  float lambda;
  float window[11];
  float* dx;             // may be null
  double* partials;      // [blocks][2]
  uint32_t* counter;     // zero between calls
  double* out;           // {loss, l1, ssim}
};

// The loss runs one CTA per channel and strip of kLossCols columns x
// kLossStrip rows (kLossStrip a multiple of 16; a build-time tunable). At
// 1920x1080, 192 rows give 1,080 CTAs, just under two waves of 4 per SM on
// 148 SMs, with a 20-row pipeline fill per strip (measured: 0.175 ms against
// 0.186 ms for 128 rows, 0.187 for 176 and 0.183 for 368).
#ifndef GS_LOSS_STRIP
#define GS_LOSS_STRIP 192
#endif
constexpr int kLossCols = 32;
constexpr int kLossStrip = GS_LOSS_STRIP;
static_assert(kLossStrip % 16 == 0, "loss strip");
constexpr int64_t loss_blocks(int height, int width) {
  return 3 * static_cast<int64_t>((width + kLossCols - 1) / kLossCols) *
         ((height + kLossStrip - 1) / kLossStrip);
}

cudaError_t launch_loss(const LossArgs& a, cudaStream_t st);

// The Charbonnier + exposure loss: out = {loss, dL/dgain[3], dL/dbias[3]}.
struct CharbonnierArgs {
  const float* x;
  const float* y;
  int64_t pixels;  // H W
  float gain[3], bias[3], delta;
  float* dx;           // may be null
  double* partials;    // [blocks][7]
  uint32_t* counter;   // zero between calls
  double* out;         // [7]
};
constexpr int kCharbMaxBlocks = 148 * 8;
int charbonnier_blocks(int64_t pixels);
cudaError_t launch_charbonnier(const CharbonnierArgs& a, cudaStream_t st);

// ------------------------------------------------------- projection backward
struct PreprocessBwdArgs {
  const float *means, *log_scales, *quats, *opacity_logits, *sh;
  int64_t n, n_pad;
  int sh_k, active_degree;
  CamArgs cam;
  const Screen* screen;
  const uint32_t* touched;
  const uint8_t* clamped;
  const float* sgrad;
  float *g_means, *g_log_scales, *g_quats, *g_opacity_logits, *g_sh;
  // density-control statistics (both null when not accumulating)
  float* stat_accum;
  uint32_t* stat_count;
  int mip_comp;  // the screen opacity includes the compensation factor (GS_OPTION_MIP_COMPENSATION)
};

cudaError_t launch_preprocess_backward(const PreprocessBwdArgs& a, cudaStream_t st);

// Camera-pose gradient of one view: out = {dL/dw (3), dL/dt (3)} in float64,
// from the same per-Gaussian inputs as the projection backward.
constexpr int kCamBlocks = 148 * 3;
struct CameraGradArgs {
  double* out;       // [6], device
  double* partials;  // [kCamBlocks][9]
  uint32_t* counter; // zero between calls (the last CTA resets it)
};
cudaError_t launch_camera_backward(const PreprocessBwdArgs& a, const CameraGradArgs& g, cudaStream_t st);

// Parameters (written in place), accumulated gradients (zeroed), Adam moments
// and per-group scalars, in group order means, log_scales, quats,
// opacity_logits, sh.
struct FusedAdamArgs {
  float* p[5];
  float* g[5];
  float* m[5];
  float* v[5];
  AdamScalars s[5];
};

cudaError_t launch_preprocess_backward_adam(const PreprocessBwdArgs& a, const FusedAdamArgs& f,
                                           cudaStream_t st);
AdamScalars adam_scalars(float lr, float beta1, float beta2, float eps, int step);
cudaError_t launch_screen_grads(const Screen* screen, const float* sgrad, int64_t n, float* out,
                                cudaStream_t st);

// ------------------------------------------------------- density control
struct DensifyArgs {
  const float *means, *log_scales, *quats, *opacity_logits, *sh;  // in, planar with stride np_in
  const float *m[5], *v[5];                                       // moments in, same layout
  int64_t n, np_in;
  int sh_k;
  const float* grad_accum;
  const uint32_t* view_count;
  const float* normals;  // [n][2][3]
  double grad_threshold, log_scale_threshold, logit_threshold;
  float *out_p[5], *out_m[5], *out_v[5];  // planar with stride np_out
  int64_t np_out;
  uint4* block_counts;   // [blocks]: kept, clones, splits
  uint4* block_prefix;   // [blocks]: exclusive prefixes of the same
  uint4* totals;         // [1]
};
constexpr int kDensifyBlock = 256;
cudaError_t launch_densify_count(const DensifyArgs& a, cudaStream_t st);
cudaError_t launch_densify_write(const DensifyArgs& a, uint4 totals, cudaStream_t st);
cudaError_t launch_opacity_reset(float* logits, float* m, float* v, int64_t n, float cap, cudaStream_t st);

// Recycling dead Gaussians onto the largest donors, in place (count fixed).
struct RelocateArgs {
  float* p[5];  // means, log_scales, quats, opacity_logits, sh: planar with stride np, updated in place
  float* m[5];  // Adam moments, same layout
  float* v[5];
  int64_t n, np;
  int sh_k;
  double dead_logit, donor_logit;  // logit < dead_logit: dead; logit > donor_logit: donor
  uint4* block_counts;             // [blocks]: dead, donors
  uint4* block_prefix;             // [blocks]: exclusive prefixes of the same
  uint4* totals;                   // [1]
  uint32_t* dead;                  // [n]: dead indices in index order
  uint32_t* donor_keys;            // [n]: sort keys, largest log-scale first
  uint32_t* donor_vals;            // [n]: donor indices in index order
  const uint32_t* sorted_donors;   // the donor indices after the (stable) sort
  const float* normals;            // [pairs][3] N(0, 1) draws
  int64_t pairs;
  uint32_t* err;
};
cudaError_t launch_relocate_classify(const RelocateArgs& a, cudaStream_t st);
cudaError_t launch_relocate_pairs(const RelocateArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- Adam
cudaError_t launch_adam(float* p, float* g, float* m, float* v, int64_t count, float lr,
                        float beta1, float beta2, float eps, int step, cudaStream_t st);

// ------------------------------------------- data-parallel exchange + Adam
constexpr int kMaxRanks = 8;  // GPUs of one NVSwitch node

struct ReduceAdamArgs {
  float* p;  // this rank's shard: parameters and moments, updated in place
  float* m;
  float* v;
  int64_t count;
  float* grads[kMaxRanks];   // every rank's gradient at this shard (local or peer memory)
  int n_grads;
  float* copies[kMaxRanks];  // other ranks' parameter buffers at this shard (peer memory)
  int n_copies;
  int zero_grads;            // write zeros to every gradient source after reading it
  float grad_scale;          // 1 / ranks: the mean gradient
  AdamScalars s;
};

cudaError_t launch_adam_reduce(const ReduceAdamArgs& a, cudaStream_t st);

// ------------------------------- data-parallel update from the views' sums
// One rank's view of the Gaussians after its blend backward (device pointers,
// local or peer memory): screen records, raw screen-gradient sums, touched and
// clamp flags, and its camera record.
struct ViewArgs {
  const Screen* screen;
  const float* sgrad;
  const uint32_t* touched;
  const uint8_t* clamped;
  const CamArgs* cam;
};

struct ViewsAdamArgs {
  PreprocessBwdArgs base;  // this rank's parameters, sizes and options (view fields unused)
  ViewArgs views[kMaxRanks];
  int n_views;
  int64_t g_lo, g_hi;      // this rank's Gaussians [g_lo, g_hi), multiples of 4
  FusedAdamArgs f;         // parameters (updated in place), moments, per-group scalars
  float* copies[kMaxRanks][5];  // other ranks' parameter groups (peer memory)
  int n_copies;
  float grad_scale;        // 1 / ranks: the batch mean
};
cudaError_t launch_views_adam(const ViewsAdamArgs& a, cudaStream_t st);

}  // namespace gs
