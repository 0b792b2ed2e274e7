// Kernel argument records and host-side launchers of the rasteriser stages.
// Everything here is internal to the library; the public surface is gs_api.h.
#pragma once

#include "adam_math.cuh"
#include "gs_common.cuh"

namespace gs {

// Written by the preprocess + block scan and read back by the host before the
// sort: the entry count and the range of depth keys of visible Gaussians.
struct ForwardInfo {
  uint64_t num_entries;
  uint32_t depth_min, depth_max;
  uint32_t device_error;
  uint32_t pad;
};

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
  uint32_t* block_sums;   // one per 256-Gaussian block
  uint32_t* depth_range;  // [min, max] of visible depth keys (atomics)
};

cudaError_t launch_preprocess(const PreprocessArgs& a, int64_t num_blocks, cudaStream_t st);
cudaError_t launch_scan_blocks(const uint32_t* block_sums, int64_t num_blocks, uint64_t* block_prefix,
                               const uint32_t* depth_range, ForwardInfo* info, cudaStream_t st);

// ---------------------------------------------------------------- sorting
struct SortPlan {
  int64_t n;       // entries
  int depth_bits;  // bits kept of (depth key - depth_min)
  int key_bits;    // tile bits + depth_bits
  int passes;      // ceil(key_bits / 8)
  int64_t tiles;   // onesweep tiles of kSortTileKeys entries
};

constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortTileKeys = kSortThreads * kSortItems;  // 4096
constexpr int kRadix = 256;
constexpr int kMaxPasses = 8;

struct DuplicateArgs {
  int64_t n;
  const uint32_t* touched;
  const uint2* rect;
  const float* depth;
  const uint64_t* block_prefix;
  uint32_t depth_min;
  int depth_bits;
  int tiles_x;
  int64_t max_entries;
  uint64_t* keys;
  uint32_t* vals;
  uint32_t* err;
};

cudaError_t launch_duplicate(const DuplicateArgs& a, int64_t num_blocks, cudaStream_t st);

struct SortBuffers {
  uint64_t* keys[2];
  uint32_t* vals[2];
  uint32_t* hist;      // [kMaxPasses][256] digit counts
  uint32_t* offsets;   // [kMaxPasses][256] exclusive digit offsets
  uint32_t* status;    // [kMaxPasses][tiles][256] look-back words
  uint32_t* counters;  // [kMaxPasses] tile tickets
  uint32_t* err;
};

// Sorts keys[0]/vals[0]; returns in *out_buf the buffer (0 or 1) holding the result.
cudaError_t launch_sort(const SortPlan& plan, const SortBuffers& b, int* out_buf, cudaStream_t st);

cudaError_t launch_ranges(const uint64_t* keys, int64_t n, int depth_bits, uint2* ranges,
                          int64_t num_tiles, cudaStream_t st);

// ---------------------------------------------------------------- blending
struct BlendArgs {
  const uint2* ranges;
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
};

cudaError_t launch_blend_forward(const BlendArgs& a, cudaStream_t st);
cudaError_t launch_blend_backward(const BlendArgs& a, cudaStream_t st);

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

cudaError_t launch_loss(const LossArgs& a, cudaStream_t st);

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
};

cudaError_t launch_preprocess_backward(const PreprocessBwdArgs& a, cudaStream_t st);

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

// ---------------------------------------------------------------- Adam
cudaError_t launch_adam(float* p, float* g, float* m, float* v, int64_t count, float lr,
                        float beta1, float beta2, float eps, int step, cudaStream_t st);

}  // namespace gs
