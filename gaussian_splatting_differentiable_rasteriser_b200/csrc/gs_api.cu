// C ABI of the rasteriser (declared in include/gs_api.h): context management,
// host-side argument checks and the order of kernel launches per call.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "gs_api.h"
#include "gs_kernels.cuh"

namespace gs {
int64_t loss_num_blocks(int height, int width);
}

struct gs_ctx {
  int64_t max_g = 0, max_k = 0, max_tiles = 0, max_blocks = 0, max_sort_tiles = 0,
          max_loss_blocks = 0;
  int32_t max_w = 0, max_h = 0;
  // per Gaussian
  gs::Screen* screen = nullptr;
  gs::CamArgs* cam_dev = nullptr;  // the camera of the last blend backward (data-parallel views)
  bool have_view = false;
  float* depth = nullptr;
  uint2* rect = nullptr;
  uint32_t* touched = nullptr;
  uint8_t* clamped = nullptr;
  float* sgrad = nullptr;
  uint2* block_sums = nullptr;
  uint32_t* visible_prefix = nullptr;
  uint32_t* depth_range = nullptr;
  // depth sort of the visible Gaussians
  uint32_t* dkeys[2] = {nullptr, nullptr};
  uint32_t* dvals[2] = {nullptr, nullptr};
  uint32_t* dup_offsets = nullptr;
  // tile sort of the entries
  uint32_t* keys[2] = {nullptr, nullptr};
  uint32_t* vals[2] = {nullptr, nullptr};
  uint32_t* hist = nullptr;
  uint32_t* offsets = nullptr;
  uint32_t* chunk_counts = nullptr;
  uint2* ranges = nullptr;
  uint32_t* tile_order = nullptr;  // [max_tiles] tiles by descending list length
  uint2* surv = nullptr;           // [8][max_entries]: per-warp survivors of the blend's box test
  uint32_t* surv_count = nullptr;  // [max_tiles][8]
  // loss
  double* loss_partials = nullptr;
  uint32_t* loss_counter = nullptr;
  double* charb_partials = nullptr;  // [kCharbMaxBlocks][7]
  uint32_t* charb_counter = nullptr;
  // camera-pose gradient: caller's output (NULL when off) and the kernel's scratch
  double* cam_out = nullptr;
  uint32_t* reloc_dead = nullptr;  // [max_g], allocated by the first gs_relocate
  double* cam_partials = nullptr;  // [kCamBlocks][9]
  uint32_t* cam_counter = nullptr;
  // readback record (device + pinned host); the device error word lives in it
  gs::ForwardInfo* info_dev = nullptr;
  gs::ForwardInfo* info_host = nullptr;
  // state of the camera in flight
  bool have_pre = false, have_fwd = false;
  // The screen-gradient sums (float32, or fixed point in deterministic mode)
  // are zeroed by gs_render_forward while the host waits for the entry count;
  // the backward zeroes them itself when these are false.
  bool sgrad_zeroed = false, sgrad_fixed_zeroed = false;
  cudaEvent_t info_ev = nullptr;  // the entry count has reached the host
  int64_t n = 0, n_pad = 0;
  gs::CamArgs cam{};
  int64_t K = 0;
  int sorted_buf = 0;
  // options (gs_set_option)
  int opacity_rect = 0;
  int mip_comp = 0;
  unsigned long long* sgrad_fixed = nullptr;  // [max_g][9], allocated by GS_OPTION_DETERMINISTIC
  int deterministic = 0;
  // density control: caller-owned statistics buffers, and the pass's scratch
  float* stat_accum = nullptr;
  uint32_t* stat_count = nullptr;
  uint4* dens_counts = nullptr;  // [max_blocks]
  uint4* dens_prefix = nullptr;  // [max_blocks]
  uint4* dens_totals = nullptr;  // [1], device
  uint4* dens_host = nullptr;    // [1], pinned host
  // profiling (off by default)
  struct Profiler {
    static constexpr int kMaxRec = 128;
    bool on = false, count = false, created = false;
    cudaEvent_t ev[2 * kMaxRec];
    int stage[kMaxRec];
    int nrec = 0;
    double ms[GS_NUM_STAGES] = {0};
    int64_t launches[GS_NUM_STAGES] = {0};
    int64_t work[GS_NUM_STAGES] = {0};
  } prof;
  unsigned long long* pairs = nullptr;  // [8]: forward at [0], [2]; backward at [4], [6]
  char err[512] = {0};
};

namespace {

gs_status fail(gs_ctx* c, gs_status s, const char* fmt, ...) {
  if (c) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(c->err, sizeof(c->err), fmt, ap);
    va_end(ap);
  }
  return s;
}

#define GS_CUDA(ctx, call)                                                              \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail((ctx), GS_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

void free_all(gs_ctx* c) {
  void* bufs[] = {c->screen, c->depth, c->rect, c->touched, c->clamped, c->sgrad, c->block_sums,
                  c->visible_prefix, c->depth_range, c->dkeys[0], c->dkeys[1], c->dvals[0],
                  c->dvals[1], c->dup_offsets, c->keys[0], c->keys[1], c->vals[0], c->vals[1],
                  c->hist, c->offsets, c->chunk_counts, c->ranges, c->tile_order, c->surv, c->surv_count,
                  c->sgrad_fixed, c->dens_counts, c->dens_prefix, c->dens_totals, c->charb_partials,
                  c->charb_counter, c->cam_partials, c->cam_counter, c->reloc_dead, c->loss_partials,
                  c->loss_counter, c->info_dev, c->pairs, c->cam_dev};
  for (void* b : bufs)
    if (b) cudaFree(b);
  if (c->info_host) cudaFreeHost(c->info_host);
  if (c->dens_host) cudaFreeHost(c->dens_host);
  if (c->prof.created)
    for (auto& e : c->prof.ev) cudaEventDestroy(e);
  if (c->info_ev) cudaEventDestroy(c->info_ev);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

gs_status make_cam(gs_ctx* c, const gs_camera* cam, gs::CamArgs& out) {
  if (!cam) return fail(c, GS_ERR_INVALID_ARG, "camera is NULL");
  if (cam->width <= 0 || cam->height <= 0 || cam->width > c->max_w || cam->height > c->max_h)
    return fail(c, GS_ERR_INVALID_ARG, "camera %dx%d outside the context's 1..%dx1..%d", cam->width,
                cam->height, c->max_w, c->max_h);
  if (!(std::isfinite(cam->fx) && std::isfinite(cam->fy) && cam->fx > 0.f && cam->fy > 0.f))
    return fail(c, GS_ERR_INVALID_ARG, "focal lengths must be finite and positive");
  out.width = cam->width;
  out.height = cam->height;
  out.tiles_x = (cam->width + gs::kTile - 1) / gs::kTile;
  out.tiles_y = (cam->height + gs::kTile - 1) / gs::kTile;
  out.fx = cam->fx;
  out.fy = cam->fy;
  out.cx = cam->cx;
  out.cy = cam->cy;
  std::memcpy(out.R, cam->R, sizeof(out.R));
  std::memcpy(out.t, cam->t, sizeof(out.t));
  std::memcpy(out.campos, cam->campos, sizeof(out.campos));
  std::memcpy(out.bg, cam->bg, sizeof(out.bg));
  out.near_z = cam->near_z;
  return GS_OK;
}

gs_status check_params(gs_ctx* c, const gs_params* p) {
  if (!p) return fail(c, GS_ERR_INVALID_ARG, "params is NULL");
  if (p->n < 0 || p->n > c->max_g)
    return fail(c, GS_ERR_INVALID_ARG, "n = %lld outside 0..%lld", (long long)p->n, (long long)c->max_g);
  if (p->n_pad < p->n || p->n_pad % 4 != 0)
    return fail(c, GS_ERR_INVALID_ARG, "n_pad = %lld must be >= n and a multiple of 4", (long long)p->n_pad);
  if (p->sh_degree < 0 || p->sh_degree > 3 || p->active_degree < 0 || p->active_degree > p->sh_degree)
    return fail(c, GS_ERR_INVALID_ARG, "sh_degree %d / active_degree %d out of range", p->sh_degree,
                p->active_degree);
  const void* ptrs[] = {p->means, p->log_scales, p->quats, p->opacity_logits, p->sh};
  if (p->n > 0)
    for (const void* q : ptrs)
      if (!q || !aligned(q, 16))
        return fail(c, GS_ERR_INVALID_ARG, "a parameter pointer is NULL or not 16-byte aligned");
  return GS_OK;
}

gs_status take_device_error(gs_ctx* c) {
  const uint32_t e = c->info_host->device_error;
  if (e == 0) return GS_OK;
  c->info_host->device_error = 0;
  cudaMemset(&c->info_dev->device_error, 0, sizeof(uint32_t));
  return fail(c, GS_ERR_DEVICE, "a kernel recorded a device fault (code 0x%x: %s)", e,
              (e & gs::kErrCopyTimeout) ? "parameter copy wait gave up" : "index out of range");
}

void prof_harvest(gs_ctx* c) {
  auto& P = c->prof;
  for (int r = 0; r < P.nrec; ++r) {
    float ms = 0.f;
    if (cudaEventSynchronize(P.ev[2 * r + 1]) == cudaSuccess &&
        cudaEventElapsedTime(&ms, P.ev[2 * r], P.ev[2 * r + 1]) == cudaSuccess)
      P.ms[P.stage[r]] += ms;
  }
  P.nrec = 0;
}

void prof_begin(gs_ctx* c, cudaStream_t st) {
  auto& P = c->prof;
  if (!P.on) return;
  if (P.nrec == gs_ctx::Profiler::kMaxRec) prof_harvest(c);
  cudaEventRecord(P.ev[2 * P.nrec], st);
}

// Closes a timed bracket of `kernels` kernel launches doing `work` units.
void prof_end(gs_ctx* c, int stage, int64_t work, cudaStream_t st, int kernels = 1) {
  auto& P = c->prof;
  if (!P.on) return;
  cudaEventRecord(P.ev[2 * P.nrec + 1], st);
  P.stage[P.nrec++] = stage;
  P.launches[stage] += kernels;
  P.work[stage] += work;
}

// Kernels one launch_sort enqueues: upsweep, digit scan and downsweep per pass.
int sort_kernels(const gs::SortPlan& p) { return (p.n > 1 && p.passes > 0) ? 3 * p.passes : 0; }

__global__ void unpack_preprocess_kernel(const gs::Screen* screen, const float* depth,
                                         const uint2* rect, const uint32_t* touched,
                                         const uint8_t* clamped, int64_t n, float* mean2d,
                                         float* conic, float* opacity, float* rgb, float* dep,
                                         int32_t* rc, int32_t* tt, uint8_t* cl) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const gs::Screen s = screen[i];
  if (mean2d) {
    mean2d[2 * i] = s.a.x;
    mean2d[2 * i + 1] = s.a.y;
  }
  if (conic) {
    conic[3 * i] = gs::conic_A(s);
    conic[3 * i + 1] = gs::conic_B(s);
    conic[3 * i + 2] = gs::conic_C(s);
  }
  if (opacity) opacity[i] = gs::screen_opacity(s);
  if (rgb) {
    rgb[3 * i] = s.c.x;
    rgb[3 * i + 1] = s.c.y;
    rgb[3 * i + 2] = s.c.z;
  }
  if (dep) dep[i] = depth[i];
  if (rc) {
    const uint2 r = rect[i];
    rc[4 * i] = static_cast<int32_t>(r.x & 0xffffu);
    rc[4 * i + 1] = static_cast<int32_t>(r.y & 0xffffu);
    rc[4 * i + 2] = static_cast<int32_t>(r.x >> 16);
    rc[4 * i + 3] = static_cast<int32_t>(r.y >> 16);
  }
  if (tt) tt[i] = static_cast<int32_t>(touched[i]);
  if (cl) cl[i] = clamped[i];
}

int bit_length(uint64_t v) { return v == 0 ? 0 : 64 - __builtin_clzll(v); }

}  // namespace

extern "C" {

gs_status gs_create(gs_ctx** out, int64_t max_gaussians, int64_t max_entries, int32_t max_width,
                    int32_t max_height) {
  if (!out) return GS_ERR_INVALID_ARG;
  *out = nullptr;
  if (max_gaussians <= 0 || max_entries <= 0 || max_width <= 0 || max_height <= 0 ||
      max_gaussians > (int64_t(1) << 31) - 1 || max_entries >= (int64_t(1) << 30) ||
      max_width > 16 * 65535 || max_height > 16 * 65535)
    return GS_ERR_INVALID_ARG;
  gs_ctx* c = new gs_ctx();
  c->max_g = max_gaussians;
  c->max_k = max_entries;
  c->max_w = max_width;
  c->max_h = max_height;
  c->max_tiles = static_cast<int64_t>((max_width + 15) / 16) * ((max_height + 15) / 16);
  c->max_blocks = (max_gaussians + gs::kGaussBlock - 1) / gs::kGaussBlock;
  // the depth sort (visible Gaussians) and the tile sort (entries) share the per-chunk digit counts
  c->max_sort_tiles = (std::max(max_entries, max_gaussians) + gs::kSortTileKeys - 1) / gs::kSortTileKeys;
  c->max_loss_blocks = gs::loss_num_blocks(max_height, max_width);
  const int64_t G = max_gaussians, K = max_entries;
  cudaError_t e = cudaSuccess;
#define GS_ALLOC(ptr, bytes) \
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&(ptr)), (bytes))
  GS_ALLOC(c->screen, sizeof(gs::Screen) * G);
  GS_ALLOC(c->cam_dev, sizeof(gs::CamArgs));
  GS_ALLOC(c->depth, sizeof(float) * G);
  GS_ALLOC(c->rect, sizeof(uint2) * G);
  GS_ALLOC(c->touched, sizeof(uint32_t) * G);
  GS_ALLOC(c->clamped, sizeof(uint8_t) * G);
  GS_ALLOC(c->sgrad, sizeof(float) * gs::kGradStride * G);
  GS_ALLOC(c->block_sums, sizeof(uint2) * c->max_blocks);
  GS_ALLOC(c->visible_prefix, sizeof(uint32_t) * c->max_blocks);
  GS_ALLOC(c->depth_range, sizeof(uint32_t) * 2);
  GS_ALLOC(c->dkeys[0], sizeof(uint32_t) * G);
  GS_ALLOC(c->dkeys[1], sizeof(uint32_t) * G);
  GS_ALLOC(c->dvals[0], sizeof(uint32_t) * G);
  GS_ALLOC(c->dvals[1], sizeof(uint32_t) * G);
  GS_ALLOC(c->dup_offsets, sizeof(uint32_t) * ((G + gs::kDupItems - 1) / gs::kDupItems));
  GS_ALLOC(c->keys[0], sizeof(uint32_t) * K);
  GS_ALLOC(c->keys[1], sizeof(uint32_t) * K);
  GS_ALLOC(c->vals[0], sizeof(uint32_t) * K);
  GS_ALLOC(c->vals[1], sizeof(uint32_t) * K);
  GS_ALLOC(c->hist, sizeof(uint32_t) * gs::kMaxPasses * gs::kRadix);
  GS_ALLOC(c->offsets, sizeof(uint32_t) * gs::kMaxPasses * gs::kRadix);
  GS_ALLOC(c->chunk_counts, sizeof(uint32_t) * gs::kMaxPasses * gs::kRadix * c->max_sort_tiles);
  GS_ALLOC(c->ranges, sizeof(uint2) * c->max_tiles);
  GS_ALLOC(c->tile_order, sizeof(uint32_t) * c->max_tiles);
  GS_ALLOC(c->surv, sizeof(uint2) * 8 * K);
  GS_ALLOC(c->surv_count, sizeof(uint32_t) * 8 * c->max_tiles);
  GS_ALLOC(c->dens_counts, sizeof(uint4) * ((G + gs::kDensifyBlock - 1) / gs::kDensifyBlock));
  GS_ALLOC(c->dens_prefix, sizeof(uint4) * ((G + gs::kDensifyBlock - 1) / gs::kDensifyBlock));
  GS_ALLOC(c->dens_totals, sizeof(uint4));
  GS_ALLOC(c->loss_partials, sizeof(double) * 2 * c->max_loss_blocks);
  GS_ALLOC(c->loss_counter, sizeof(uint32_t));
  GS_ALLOC(c->charb_partials, sizeof(double) * 7 * gs::kCharbMaxBlocks);
  GS_ALLOC(c->charb_counter, sizeof(uint32_t));
  GS_ALLOC(c->cam_partials, sizeof(double) * 9 * gs::kCamBlocks);
  GS_ALLOC(c->cam_counter, sizeof(uint32_t));
  GS_ALLOC(c->info_dev, sizeof(gs::ForwardInfo));
  GS_ALLOC(c->pairs, sizeof(unsigned long long) * 8);
#undef GS_ALLOC
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c->info_ev, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaMallocHost(reinterpret_cast<void**>(&c->info_host), sizeof(gs::ForwardInfo));
  if (e == cudaSuccess) e = cudaMallocHost(reinterpret_cast<void**>(&c->dens_host), sizeof(uint4));
  if (e == cudaSuccess) e = cudaMemset(c->loss_counter, 0, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(c->charb_counter, 0, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(c->cam_counter, 0, sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMemset(c->info_dev, 0, sizeof(gs::ForwardInfo));
  if (e == cudaSuccess) e = cudaMemset(c->pairs, 0, sizeof(unsigned long long) * 8);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    free_all(c);
    delete c;
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  std::memset(c->info_host, 0, sizeof(gs::ForwardInfo));
  *out = c;
  return GS_OK;
}

void gs_destroy(gs_ctx* ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  free_all(ctx);
  delete ctx;
}

const char* gs_last_error(const gs_ctx* ctx) { return ctx ? ctx->err : "no context"; }

gs_status gs_set_option(gs_ctx* c, int32_t option, int32_t value) {
  if (!c) return GS_ERR_INVALID_ARG;
  switch (option) {
    case GS_OPTION_OPACITY_RECT:
      if (value != 0 && value != 1) return fail(c, GS_ERR_INVALID_ARG, "option value must be 0 or 1");
      c->opacity_rect = value;
      c->have_pre = c->have_fwd = false;  // the tile lists depend on it
      return GS_OK;
    case GS_OPTION_MIP_COMPENSATION:
      if (value != 0 && value != 1) return fail(c, GS_ERR_INVALID_ARG, "option value must be 0 or 1");
      c->mip_comp = value;
      c->have_pre = c->have_fwd = false;  // the screen opacities depend on it
      return GS_OK;
    case GS_OPTION_DETERMINISTIC:
      if (value != 0 && value != 1) return fail(c, GS_ERR_INVALID_ARG, "option value must be 0 or 1");
      if (value && !c->sgrad_fixed)
        GS_CUDA(c, cudaMalloc(reinterpret_cast<void**>(&c->sgrad_fixed),
                              sizeof(unsigned long long) * gs::kFixedStride * c->max_g));
      c->deterministic = value;
      return GS_OK;
    default:
      return fail(c, GS_ERR_INVALID_ARG, "unknown option %d", option);
  }
}

gs_status gs_preprocess(gs_ctx* c, const gs_params* p, const gs_camera* cam, void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  gs_status s = check_params(c, p);
  if (s != GS_OK) return s;
  gs::CamArgs ca;
  if ((s = make_cam(c, cam, ca)) != GS_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  c->have_pre = c->have_fwd = false;
  GS_CUDA(c, cudaMemsetAsync(c->depth_range, 0xff, sizeof(uint32_t), st));
  GS_CUDA(c, cudaMemsetAsync(c->depth_range + 1, 0, sizeof(uint32_t), st));
  gs::PreprocessArgs a;
  a.means = p->means;
  a.log_scales = p->log_scales;
  a.quats = p->quats;
  a.opacity_logits = p->opacity_logits;
  a.sh = p->sh;
  a.n = p->n;
  a.n_pad = p->n_pad;
  a.sh_k = (p->sh_degree + 1) * (p->sh_degree + 1);
  a.active_degree = p->active_degree;
  a.cam = ca;
  a.screen = c->screen;
  a.depth = c->depth;
  a.rect = c->rect;
  a.touched = c->touched;
  a.clamped = c->clamped;
  a.block_sums = c->block_sums;
  a.depth_range = c->depth_range;
  a.err = &c->info_dev->device_error;
  a.opacity_rect = c->opacity_rect;
  a.mip_comp = c->mip_comp;
  const int64_t nb = (p->n + gs::kGaussBlock - 1) / gs::kGaussBlock;
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_preprocess(a, nb, st));
  prof_end(c, GS_STAGE_PREPROCESS, p->n, st, p->n > 0 ? 1 : 0);
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_scan_blocks(c->block_sums, nb, c->visible_prefix, c->depth_range, c->info_dev, st));
  prof_end(c, GS_STAGE_SCAN, nb, st);
  c->n = p->n;
  c->n_pad = p->n_pad;
  c->cam = ca;
  c->have_pre = true;
  return GS_OK;
}

gs_status gs_render_forward(gs_ctx* c, const gs_camera* cam, float* image, float* final_T,
                            int32_t* n_contrib, int64_t* num_entries_out, void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (!c->have_pre) return fail(c, GS_ERR_INVALID_ARG, "gs_preprocess has not run");
  gs::CamArgs ca;
  gs_status s = make_cam(c, cam, ca);
  if (s != GS_OK) return s;
  if (ca.width != c->cam.width || ca.height != c->cam.height)
    return fail(c, GS_ERR_INVALID_ARG, "camera size differs from the one preprocessed");
  if (!image || !final_T || !n_contrib || !aligned(image, 4) || !aligned(final_T, 4) ||
      !aligned(n_contrib, 4))
    return fail(c, GS_ERR_INVALID_ARG, "output pointers must be non-NULL and 4-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  c->have_fwd = false;
  // The one host/device crossing of the step: entry count and depth-key range.
  GS_CUDA(c, cudaMemcpyAsync(c->info_host, c->info_dev, sizeof(gs::ForwardInfo),
                             cudaMemcpyDeviceToHost, st));
  GS_CUDA(c, cudaEventRecord(c->info_ev, st));
  // The backward's screen-gradient sums are cleared now: the device does it
  // while the host waits for the counts, and the backward then needs no
  // memset between the loss and the blend backward.
  c->sgrad_zeroed = c->sgrad_fixed_zeroed = false;
  if (c->n > 0) {
    if (c->deterministic)
      GS_CUDA(c, cudaMemsetAsync(c->sgrad_fixed, 0, sizeof(unsigned long long) * gs::kFixedStride * c->n, st));
    else
      GS_CUDA(c, cudaMemsetAsync(c->sgrad, 0, sizeof(float) * gs::kGradStride * c->n, st));
    (c->deterministic ? c->sgrad_fixed_zeroed : c->sgrad_zeroed) = true;
  }
  GS_CUDA(c, cudaEventSynchronize(c->info_ev));
  if ((s = take_device_error(c)) != GS_OK) return s;
  const uint64_t K = c->info_host->num_entries;
  if (num_entries_out) *num_entries_out = static_cast<int64_t>(K);
  if (K > static_cast<uint64_t>(c->max_k))
    return fail(c, GS_ERR_CAPACITY, "%llu (Gaussian, tile) entries exceed the context's %lld",
                (unsigned long long)K, (long long)c->max_k);
  const int64_t tiles = static_cast<int64_t>(ca.tiles_x) * ca.tiles_y;
  const int64_t V = static_cast<int64_t>(c->info_host->num_visible);
  int sorted = 0;
  if (K > 0) {
    gs::SortBuffers b;
    b.hist = c->hist;
    b.offsets = c->offsets;
    b.chunk_counts = c->chunk_counts;
    b.err = &c->info_dev->device_error;
    // 1 + 2. visible Gaussians in index order, sorted by depth key
    const uint32_t dmin = c->info_host->depth_min;
    gs::CompactArgs ca2;
    ca2.n = c->n;
    ca2.touched = c->touched;
    ca2.depth = c->depth;
    ca2.visible_prefix = c->visible_prefix;
    ca2.depth_min = dmin;
    ca2.max_out = c->max_g;
    ca2.keys = c->dkeys[0];
    ca2.vals = c->dvals[0];
    ca2.err = &c->info_dev->device_error;
    gs::SortPlan dplan;
    dplan.n = V;
    dplan.key_bits = bit_length(c->info_host->depth_max - dmin);
    dplan.passes = (dplan.key_bits + 7) / 8;
    dplan.tiles = (V + gs::kSortTileKeys - 1) / gs::kSortTileKeys;
    b.keys[0] = c->dkeys[0];
    b.keys[1] = c->dkeys[1];
    b.vals[0] = c->dvals[0];
    b.vals[1] = c->dvals[1];
    int dsorted = 0;
    prof_begin(c, st);
    GS_CUDA(c, gs::launch_compact(ca2, (c->n + gs::kGaussBlock - 1) / gs::kGaussBlock, st));
    GS_CUDA(c, gs::launch_sort(dplan, b, &dsorted, st));
    prof_end(c, GS_STAGE_DEPTH_SORT, dplan.n > 1 ? dplan.n * dplan.passes : 0, st,
             (c->n > 0 ? 1 : 0) + sort_kernels(dplan));
    // 3. one (tile, index) entry per touched tile, in depth order
    gs::DuplicateArgs d;
    d.count = V;
    d.order = c->dvals[dsorted];
    d.touched = c->touched;
    d.rect = c->rect;
    d.tiles_x = ca.tiles_x;
    d.max_entries = c->max_k;
    d.keys = c->keys[0];
    d.vals = c->vals[0];
    d.chunk_offsets = c->dup_offsets;
    d.err = &c->info_dev->device_error;
    prof_begin(c, st);
    GS_CUDA(c, gs::launch_duplicate(d, st));
    prof_end(c, GS_STAGE_DUPLICATE, static_cast<int64_t>(K), st, V > 0 ? 3 : 0);  // count, scan, write
    // 4. stable sort of the entries by tile
    gs::SortPlan plan;
    plan.n = static_cast<int64_t>(K);
    plan.key_bits = bit_length(static_cast<uint64_t>(tiles - 1));
    plan.passes = (plan.key_bits + 7) / 8;
    plan.tiles = (plan.n + gs::kSortTileKeys - 1) / gs::kSortTileKeys;
    b.keys[0] = c->keys[0];
    b.keys[1] = c->keys[1];
    b.vals[0] = c->vals[0];
    b.vals[1] = c->vals[1];
    prof_begin(c, st);
    GS_CUDA(c, gs::launch_sort(plan, b, &sorted, st));
    prof_end(c, GS_STAGE_SORT, plan.n > 1 ? plan.n * plan.passes : 0, st, sort_kernels(plan));
  }
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_ranges(c->keys[sorted], static_cast<int64_t>(K), c->ranges, tiles, st));
  GS_CUDA(c, gs::launch_tile_order(c->ranges, tiles, c->tile_order, st));
  prof_end(c, GS_STAGE_RANGES, static_cast<int64_t>(K), st, (K > 0 ? 1 : 0) + 1);
  gs::BlendArgs ba{};
  ba.ranges = c->ranges;
  ba.tile_order = c->tile_order;
  ba.order = c->vals[sorted];
  ba.screen = c->screen;
  ba.cam = c->cam;
  std::memcpy(ba.cam.bg, ca.bg, sizeof(ba.cam.bg));
  ba.image = image;
  ba.final_T = final_T;
  ba.n_contrib = n_contrib;
  ba.pairs = c->prof.count ? c->pairs : nullptr;
  ba.surv = c->surv;
  ba.surv_count = c->surv_count;
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_blend_forward(ba, st));
  prof_end(c, GS_STAGE_BLEND_FORWARD, 0, st);
  c->K = static_cast<int64_t>(K);
  c->sorted_buf = sorted;
  c->cam.bg[0] = ca.bg[0];
  c->cam.bg[1] = ca.bg[1];
  c->cam.bg[2] = ca.bg[2];
  c->have_fwd = true;
  return GS_OK;
}

gs_status gs_loss_l1_dssim(gs_ctx* c, const float* image, const float* target, int32_t height,
                           int32_t width, float lambda, double* loss_out, float* dloss_dimage,
                           void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (height <= 0 || width <= 0 || height > c->max_h || width > c->max_w)
    return fail(c, GS_ERR_INVALID_ARG, "image %dx%d outside the context's maximum", width, height);
  if (!image || !target || !loss_out || !aligned(image, 4) || !aligned(target, 4) ||
      !aligned(loss_out, 8) || (dloss_dimage && !aligned(dloss_dimage, 4)))
    return fail(c, GS_ERR_INVALID_ARG, "loss pointers must be non-NULL and aligned");
  if (!std::isfinite(lambda)) return fail(c, GS_ERR_INVALID_ARG, "lambda must be finite");
  gs::LossArgs a;
  a.x = image;
  a.y = target;
  a.height = height;
  a.width = width;
  a.lambda = lambda;
  double g[11], sum = 0.0;
  for (int i = 0; i < 11; ++i) sum += (g[i] = std::exp(-((i - 5) * (i - 5)) / (2.0 * 1.5 * 1.5)));
  for (int i = 0; i < 11; ++i) a.window[i] = static_cast<float>(g[i] / sum);
  a.dx = dloss_dimage;
  a.partials = c->loss_partials;
  a.counter = c->loss_counter;
  a.out = loss_out;
  prof_begin(c, static_cast<cudaStream_t>(stream));
  GS_CUDA(c, gs::launch_loss(a, static_cast<cudaStream_t>(stream)));
  prof_end(c, GS_STAGE_LOSS, static_cast<int64_t>(height) * width, static_cast<cudaStream_t>(stream));
  return GS_OK;
}

}  // extern "C"

namespace {

// Shared front half of the two backward entry points: checks, the blend
// backward, and the projection-backward argument record.
gs_status backward_common(gs_ctx* c, const gs_params* p, const gs_camera* cam, const float* final_T,
                          const int32_t* n_contrib, const float* dloss_dimage, gs_grads* g,
                          bool g_optional, cudaStream_t st, gs::PreprocessBwdArgs& a) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (!c->have_fwd) return fail(c, GS_ERR_INVALID_ARG, "gs_render_forward has not run");
  gs_status s = check_params(c, p);
  if (s != GS_OK) return s;
  if (p->n != c->n || p->n_pad != c->n_pad)
    return fail(c, GS_ERR_INVALID_ARG, "params differ from the ones preprocessed");
  gs::CamArgs ca;
  if ((s = make_cam(c, cam, ca)) != GS_OK) return s;
  if (ca.width != c->cam.width || ca.height != c->cam.height)
    return fail(c, GS_ERR_INVALID_ARG, "camera size differs from the one rendered");
  if (!final_T || !n_contrib || !dloss_dimage || (!g && !g_optional))
    return fail(c, GS_ERR_INVALID_ARG, "backward inputs must be non-NULL");
  if (g && p->n > 0) {
    float* gp[] = {g->means, g->log_scales, g->quats, g->opacity_logits, g->sh};
    for (float* q : gp)
      if (!q || !aligned(q, 4)) return fail(c, GS_ERR_INVALID_ARG, "a gradient pointer is NULL or misaligned");
  }
  if (p->n > 0) {
    if (c->deterministic && !c->sgrad_fixed_zeroed)
      GS_CUDA(c, cudaMemsetAsync(c->sgrad_fixed, 0, sizeof(unsigned long long) * gs::kFixedStride * p->n, st));
    else if (!c->deterministic && !c->sgrad_zeroed)
      GS_CUDA(c, cudaMemsetAsync(c->sgrad, 0, sizeof(float) * gs::kGradStride * p->n, st));
  }
  c->sgrad_zeroed = c->sgrad_fixed_zeroed = false;  // the blend backward adds into them
  gs::BlendArgs ba{};
  ba.ranges = c->ranges;
  ba.tile_order = c->tile_order;
  ba.order = c->vals[c->sorted_buf];
  ba.screen = c->screen;
  ba.cam = c->cam;
  ba.final_T = const_cast<float*>(final_T);
  ba.n_contrib = const_cast<int32_t*>(n_contrib);
  ba.dimage = dloss_dimage;
  ba.sgrad = c->sgrad;
  ba.pairs = c->prof.count ? c->pairs + 4 : nullptr;
  ba.surv = c->surv;
  ba.surv_count = c->surv_count;
  ba.sgrad_fixed = c->deterministic ? c->sgrad_fixed : nullptr;
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_blend_backward(ba, st));
  if (c->deterministic) GS_CUDA(c, gs::launch_decode_fixed(c->sgrad_fixed, p->n, c->sgrad, st));
  prof_end(c, GS_STAGE_BLEND_BACKWARD, 0, st, 1 + (c->deterministic && p->n > 0 ? 1 : 0));
  a.means = p->means;
  a.log_scales = p->log_scales;
  a.quats = p->quats;
  a.opacity_logits = p->opacity_logits;
  a.sh = p->sh;
  a.n = p->n;
  a.n_pad = p->n_pad;
  a.sh_k = (p->sh_degree + 1) * (p->sh_degree + 1);
  a.active_degree = p->active_degree;
  a.cam = c->cam;
  a.screen = c->screen;
  a.touched = c->touched;
  a.clamped = c->clamped;
  a.sgrad = c->sgrad;
  a.g_means = g ? g->means : nullptr;
  a.g_log_scales = g ? g->log_scales : nullptr;
  a.g_quats = g ? g->quats : nullptr;
  a.g_opacity_logits = g ? g->opacity_logits : nullptr;
  a.g_sh = g ? g->sh : nullptr;
  a.stat_accum = c->stat_accum;
  a.stat_count = c->stat_count;
  a.mip_comp = c->mip_comp;
  if (c->cam_out) {
    // camera-pose gradient of this view, from the raw sums and the parameters
    // of the render (before any update)
    prof_begin(c, st);
    if (p->n > 0) {
      gs::CameraGradArgs cg{c->cam_out, c->cam_partials, c->cam_counter};
      GS_CUDA(c, gs::launch_camera_backward(a, cg, st));
    } else {
      GS_CUDA(c, cudaMemsetAsync(c->cam_out, 0, 6 * sizeof(double), st));
    }
    prof_end(c, GS_STAGE_CAMERA_BACKWARD, p->n, st, p->n > 0 ? 1 : 0);
  }
  return GS_OK;
}

bool valid_betas(float beta1, float beta2, float eps) {
  return beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f && eps > 0.f && std::isfinite(eps);
}

}  // namespace

extern "C" {

gs_status gs_render_backward(gs_ctx* c, const gs_params* p, const gs_camera* cam, const float* final_T,
                             const int32_t* n_contrib, const float* dloss_dimage, gs_grads* g,
                             void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gs::PreprocessBwdArgs a;
  gs_status s = backward_common(c, p, cam, final_T, n_contrib, dloss_dimage, g, false, st, a);
  if (s != GS_OK) return s;
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_preprocess_backward(a, st));
  prof_end(c, GS_STAGE_PREPROCESS_BACKWARD, p->n, st, p->n > 0 ? 1 : 0);
  return GS_OK;
}

gs_status gs_render_backward_adam(gs_ctx* c, const gs_params* p, const gs_camera* cam,
                                  const float* final_T, const int32_t* n_contrib,
                                  const float* dloss_dimage, gs_grads* g, gs_grads* m, gs_grads* v,
                                  const float* lr, float beta1, float beta2, float eps, int32_t step,
                                  void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (!m || !v || !lr) return fail(c, GS_ERR_INVALID_ARG, "moments and learning rates must be non-NULL");
  if (step < 1 || !valid_betas(beta1, beta2, eps))
    return fail(c, GS_ERR_INVALID_ARG, "step must be >= 1, betas in [0, 1), eps > 0");
  for (int k = 0; k < 5; ++k)
    if (!std::isfinite(lr[k])) return fail(c, GS_ERR_INVALID_ARG, "learning rates must be finite");
  if (p && p->n_pad > 0) {
    // the fused pass moves moments (and an accumulated gradient) as float4
    float* mp[] = {m->means, m->log_scales, m->quats, m->opacity_logits, m->sh,
                   v->means, v->log_scales, v->quats, v->opacity_logits, v->sh};
    for (float* q : mp)
      if (!q || !aligned(q, 16))
        return fail(c, GS_ERR_INVALID_ARG, "a moment pointer is NULL or not 16-byte aligned");
    if (g) {
      float* gp[] = {g->means, g->log_scales, g->quats, g->opacity_logits, g->sh};
      for (float* q : gp)
        if (!q || !aligned(q, 16))
          return fail(c, GS_ERR_INVALID_ARG, "a gradient pointer is NULL or not 16-byte aligned");
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gs::PreprocessBwdArgs a;
  gs_status s = backward_common(c, p, cam, final_T, n_contrib, dloss_dimage, g, true, st, a);
  if (s != GS_OK) return s;
  gs::FusedAdamArgs f;
  const float* pp[5] = {p->means, p->log_scales, p->quats, p->opacity_logits, p->sh};
  float* gg[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
  if (g) {
    gg[0] = g->means;
    gg[1] = g->log_scales;
    gg[2] = g->quats;
    gg[3] = g->opacity_logits;
    gg[4] = g->sh;
  }
  float* mm[5] = {m->means, m->log_scales, m->quats, m->opacity_logits, m->sh};
  float* vv[5] = {v->means, v->log_scales, v->quats, v->opacity_logits, v->sh};
  for (int k = 0; k < 5; ++k) {
    f.p[k] = const_cast<float*>(pp[k]);  // documented: updated in place
    f.g[k] = gg[k];
    f.m[k] = mm[k];
    f.v[k] = vv[k];
    f.s[k] = gs::adam_scalars(lr[k], beta1, beta2, eps, step);
  }
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_preprocess_backward_adam(a, f, st));
  prof_end(c, GS_STAGE_BACKWARD_ADAM, p->n_pad, st, p->n_pad > 0 ? 1 : 0);
  return GS_OK;
}

gs_status gs_render_backward_screen(gs_ctx* c, const gs_params* p, const gs_camera* cam, const float* final_T,
                                    const int32_t* n_contrib, const float* dloss_dimage, void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gs::PreprocessBwdArgs a;
  gs_status s = backward_common(c, p, cam, final_T, n_contrib, dloss_dimage, nullptr, true, st, a);
  if (s != GS_OK) return s;
  // the camera of this view, for the ranks whose update kernels read it
  GS_CUDA(c, cudaMemcpyAsync(c->cam_dev, &c->cam, sizeof(gs::CamArgs), cudaMemcpyHostToDevice, st));
  c->have_view = true;
  return GS_OK;
}

gs_status gs_get_view(const gs_ctx* c, gs_view* out) {
  if (!c || !out) return GS_ERR_INVALID_ARG;
  out->screen = c->screen;
  out->sums = c->sgrad;
  out->touched = c->touched;
  out->clamped = c->clamped;
  out->camera = c->cam_dev;
  return GS_OK;
}

gs_status gs_shared_handle(const void* ptr, unsigned char* handle) {
  if (!ptr || !handle) return GS_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, const_cast<void*>(ptr)) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  std::memcpy(handle, &h, sizeof(h));
  return GS_OK;
}

gs_status gs_adam_step_views(gs_ctx* c, const gs_params* p, const gs_view* views, int32_t n_views, int64_t g_lo,
                             int64_t g_hi, const gs_grads* copies, int32_t n_copies, gs_grads* m, gs_grads* v,
                             const float* lr, float grad_scale, float beta1, float beta2, float eps, int32_t step,
                             void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  gs_status s = check_params(c, p);
  if (s != GS_OK) return s;
  if (!views || n_views < 1 || n_views > gs::kMaxRanks || n_copies < 0 || n_copies > gs::kMaxRanks ||
      (n_copies > 0 && !copies))
    return fail(c, GS_ERR_INVALID_ARG, "1..%d views and 0..%d copies required", gs::kMaxRanks, gs::kMaxRanks);
  if (g_lo < 0 || g_hi < g_lo || g_hi > p->n_pad || g_lo % 4 != 0 || g_hi % 4 != 0)
    return fail(c, GS_ERR_INVALID_ARG, "Gaussian range [%lld, %lld) must lie in [0, n_pad] on multiples of 4",
                (long long)g_lo, (long long)g_hi);
  if (!m || !v || !lr) return fail(c, GS_ERR_INVALID_ARG, "moments and learning rates must be non-NULL");
  if (step < 1 || !valid_betas(beta1, beta2, eps) || !std::isfinite(grad_scale))
    return fail(c, GS_ERR_INVALID_ARG, "step must be >= 1, betas in [0, 1), eps > 0, grad_scale finite");
  for (int k = 0; k < 5; ++k)
    if (!std::isfinite(lr[k])) return fail(c, GS_ERR_INVALID_ARG, "learning rates must be finite");
  gs::ViewsAdamArgs a{};
  a.base.means = p->means;
  a.base.log_scales = p->log_scales;
  a.base.quats = p->quats;
  a.base.opacity_logits = p->opacity_logits;
  a.base.sh = p->sh;
  a.base.n = p->n;
  a.base.n_pad = p->n_pad;
  a.base.sh_k = (p->sh_degree + 1) * (p->sh_degree + 1);
  a.base.active_degree = p->active_degree;
  a.base.mip_comp = c->mip_comp;
  a.n_views = n_views;
  for (int r = 0; r < n_views; ++r) {
    const gs_view& w = views[r];
    if (!w.screen || !w.sums || !w.touched || !w.clamped || !w.camera || !aligned(w.screen, 16) ||
        !aligned(w.sums, 16) || !aligned(w.touched, 4) || !aligned(w.camera, 4))
      return fail(c, GS_ERR_INVALID_ARG, "view %d has a NULL or misaligned pointer", r);
    a.views[r].screen = static_cast<const gs::Screen*>(w.screen);
    a.views[r].sgrad = w.sums;
    a.views[r].touched = w.touched;
    a.views[r].clamped = w.clamped;
    a.views[r].cam = static_cast<const gs::CamArgs*>(w.camera);
  }
  a.g_lo = g_lo;
  a.g_hi = g_hi;
  float* mm[5] = {m->means, m->log_scales, m->quats, m->opacity_logits, m->sh};
  float* vv[5] = {v->means, v->log_scales, v->quats, v->opacity_logits, v->sh};
  const float* pp[5] = {p->means, p->log_scales, p->quats, p->opacity_logits, p->sh};
  for (int k = 0; k < 5; ++k) {
    if (g_hi > g_lo && (!mm[k] || !vv[k] || !aligned(mm[k], 16) || !aligned(vv[k], 16)))
      return fail(c, GS_ERR_INVALID_ARG, "a moment pointer is NULL or not 16-byte aligned");
    a.f.p[k] = const_cast<float*>(pp[k]);  // documented: updated in place
    a.f.g[k] = nullptr;
    a.f.m[k] = mm[k];
    a.f.v[k] = vv[k];
    a.f.s[k] = gs::adam_scalars(lr[k], beta1, beta2, eps, step);
  }
  a.n_copies = n_copies;
  for (int d = 0; d < n_copies; ++d) {
    float* cp[5] = {copies[d].means, copies[d].log_scales, copies[d].quats, copies[d].opacity_logits, copies[d].sh};
    for (int k = 0; k < 5; ++k) {
      if (g_hi > g_lo && (!cp[k] || !aligned(cp[k], 16)))
        return fail(c, GS_ERR_INVALID_ARG, "copy %d has a NULL or misaligned group pointer", d);
      a.copies[d][k] = cp[k];
    }
  }
  a.grad_scale = grad_scale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_views_adam(a, st));
  prof_end(c, GS_STAGE_VIEWS_ADAM, g_hi - g_lo, st, g_hi > g_lo ? 1 : 0);
  return GS_OK;
}

gs_status gs_adam_step(float* param, float* grad, float* m, float* v, int64_t count, float lr,
                       float beta1, float beta2, float eps, int32_t step, void* stream) {
  if (count < 0 || step < 1) return GS_ERR_INVALID_ARG;
  if (count > 0 && (!param || !grad || !m || !v || !aligned(param, 4) || !aligned(grad, 4) ||
                    !aligned(m, 4) || !aligned(v, 4)))
    return GS_ERR_INVALID_ARG;
  if (!valid_betas(beta1, beta2, eps) || !std::isfinite(lr)) return GS_ERR_INVALID_ARG;
  cudaError_t e = gs::launch_adam(param, grad, m, v, count, lr, beta1, beta2, eps, step,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}

gs_status gs_adam_step_reduce(float* param, float* m, float* v, int64_t count, float* const* grads,
                              int32_t n_grads, float* const* param_copies, int32_t n_copies,
                              int32_t zero_grads, float grad_scale, float lr, float beta1, float beta2,
                              float eps, int32_t step, void* stream) {
  if (count < 0 || step < 1 || n_grads < 1 || n_grads > gs::kMaxRanks || n_copies < 0 ||
      n_copies > gs::kMaxRanks || !grads || (n_copies > 0 && !param_copies))
    return GS_ERR_INVALID_ARG;
  if (!valid_betas(beta1, beta2, eps) || !std::isfinite(lr) || !std::isfinite(grad_scale))
    return GS_ERR_INVALID_ARG;
  gs::ReduceAdamArgs a{};
  a.p = param;
  a.m = m;
  a.v = v;
  a.count = count;
  a.n_grads = n_grads;
  a.n_copies = n_copies;
  a.zero_grads = zero_grads != 0;
  a.grad_scale = grad_scale;
  a.s = gs::adam_scalars(lr, beta1, beta2, eps, step);
  for (int r = 0; r < n_grads; ++r) a.grads[r] = grads[r];
  for (int d = 0; d < n_copies; ++d) a.copies[d] = param_copies[d];
  if (count > 0) {
    if (!param || !m || !v || !aligned(param, 4) || !aligned(m, 4) || !aligned(v, 4)) return GS_ERR_INVALID_ARG;
    for (int r = 0; r < n_grads; ++r)
      if (!a.grads[r] || !aligned(a.grads[r], 4)) return GS_ERR_INVALID_ARG;
    for (int d = 0; d < n_copies; ++d)
      if (!a.copies[d] || !aligned(a.copies[d], 4)) return GS_ERR_INVALID_ARG;
  }
  const cudaError_t e = gs::launch_adam_reduce(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}

gs_status gs_shared_alloc(int64_t bytes, void** ptr, unsigned char* handle) {
  if (bytes <= 0 || !ptr || !handle) return GS_ERR_INVALID_ARG;
  *ptr = nullptr;
  void* p = nullptr;
  if (cudaMalloc(&p, static_cast<size_t>(bytes)) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  cudaIpcMemHandle_t h;
  if (cudaMemset(p, 0, static_cast<size_t>(bytes)) != cudaSuccess || cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(p);
    return GS_ERR_CUDA;
  }
  static_assert(sizeof(h) == GS_SHARED_HANDLE_BYTES, "IPC handle size");
  std::memcpy(handle, &h, sizeof(h));
  *ptr = p;
  return GS_OK;
}

gs_status gs_shared_open(const unsigned char* handle, void** ptr) {
  if (!handle || !ptr) return GS_ERR_INVALID_ARG;
  *ptr = nullptr;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  *ptr = p;
  return GS_OK;
}

gs_status gs_shared_close(void* ptr) {
  if (!ptr) return GS_ERR_INVALID_ARG;
  if (cudaIpcCloseMemHandle(ptr) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  return GS_OK;
}

gs_status gs_shared_free(void* ptr) {
  if (!ptr) return GS_ERR_INVALID_ARG;
  if (cudaFree(ptr) != cudaSuccess) {
    cudaGetLastError();
    return GS_ERR_CUDA;
  }
  return GS_OK;
}

gs_status gs_profile_enable(gs_ctx* c, int32_t enabled) {
  if (!c) return GS_ERR_INVALID_ARG;
  auto& P = c->prof;
  if (enabled && !P.created) {
    for (auto& e : P.ev) GS_CUDA(c, cudaEventCreate(&e));
    P.created = true;
  }
  if (enabled & ~(GS_PROFILE_TIME | GS_PROFILE_COUNT))
    return fail(c, GS_ERR_INVALID_ARG, "unknown profiling flags 0x%x", static_cast<unsigned>(enabled));
  if (P.on && !(enabled & GS_PROFILE_TIME)) prof_harvest(c);
  P.on = (enabled & GS_PROFILE_TIME) != 0;
  P.count = (enabled & GS_PROFILE_COUNT) != 0;
  return GS_OK;
}

gs_status gs_profile_read(gs_ctx* c, double* ms, int64_t* launches, int64_t* work,
                          int64_t* blended) {
  if (!c) return GS_ERR_INVALID_ARG;
  auto& P = c->prof;
  prof_harvest(c);
  unsigned long long pairs[8] = {0ull};
  GS_CUDA(c, cudaMemcpy(pairs, c->pairs, sizeof(pairs), cudaMemcpyDeviceToHost));
  GS_CUDA(c, cudaMemset(c->pairs, 0, sizeof(pairs)));
  P.work[GS_STAGE_BLEND_FORWARD] += static_cast<int64_t>(pairs[0]);
  P.work[GS_STAGE_BLEND_BACKWARD] += static_cast<int64_t>(pairs[4]);
  for (int k = 0; k < GS_NUM_STAGES; ++k) {
    if (ms) ms[k] = P.ms[k];
    if (launches) launches[k] = P.launches[k];
    if (work) work[k] = P.work[k];
    if (blended)
      blended[k] = k == GS_STAGE_BLEND_FORWARD ? static_cast<int64_t>(pairs[2])
                   : k == GS_STAGE_BLEND_BACKWARD ? static_cast<int64_t>(pairs[6]) : 0;
    P.ms[k] = 0.0;
    P.launches[k] = 0;
    P.work[k] = 0;
  }
  return GS_OK;
}

const char* gs_stage_name(int32_t stage) {
  static const char* names[GS_NUM_STAGES] = {"preprocess", "scan", "duplicate", "sort", "ranges",
                                             "blend_forward", "loss", "blend_backward",
                                             "preprocess_backward", "backward_adam", "depth_sort",
                                             "camera_backward", "views_adam"};
  return (stage >= 0 && stage < GS_NUM_STAGES) ? names[stage] : "";
}

gs_status gs_debug_preprocess(gs_ctx* c, float* mean2d, float* conic, float* opacity, float* rgb,
                              float* depth, int32_t* rect, int32_t* tiles_touched, uint8_t* clamped,
                              void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (!c->have_pre) return fail(c, GS_ERR_INVALID_ARG, "gs_preprocess has not run");
  if (c->n == 0) return GS_OK;
  unpack_preprocess_kernel<<<static_cast<unsigned>((c->n + 255) / 256), 256, 0,
                             static_cast<cudaStream_t>(stream)>>>(
      c->screen, c->depth, c->rect, c->touched, c->clamped, c->n, mean2d, conic, opacity, rgb, depth,
      rect, tiles_touched, clamped);
  GS_CUDA(c, cudaGetLastError());
  return GS_OK;
}

gs_status gs_debug_sorted(gs_ctx* c, int32_t* ids, int32_t* tiles, int32_t* ranges, void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (!c->have_fwd) return fail(c, GS_ERR_INVALID_ARG, "gs_render_forward has not run");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ids && c->K > 0)
    GS_CUDA(c, cudaMemcpyAsync(ids, c->vals[c->sorted_buf], sizeof(uint32_t) * c->K,
                               cudaMemcpyDeviceToDevice, st));
  if (tiles && c->K > 0)
    GS_CUDA(c, cudaMemcpyAsync(tiles, c->keys[c->sorted_buf], sizeof(uint32_t) * c->K,
                               cudaMemcpyDeviceToDevice, st));
  if (ranges)
    GS_CUDA(c, cudaMemcpyAsync(ranges, c->ranges,
                               sizeof(uint2) * static_cast<int64_t>(c->cam.tiles_x) * c->cam.tiles_y,
                               cudaMemcpyDeviceToDevice, st));
  return GS_OK;
}

gs_status gs_debug_screen_grads(gs_ctx* c, float* out, void* stream) {
  if (!c || !out) return GS_ERR_INVALID_ARG;
  if (!c->have_fwd) return fail(c, GS_ERR_INVALID_ARG, "gs_render_forward has not run");
  GS_CUDA(c, gs::launch_screen_grads(c->screen, c->sgrad, c->n, out, static_cast<cudaStream_t>(stream)));
  return GS_OK;
}


gs_status gs_set_camera_grad(gs_ctx* c, double* out) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (out && !aligned(out, 8)) return fail(c, GS_ERR_INVALID_ARG, "camera gradient output must be 8-byte aligned");
  c->cam_out = out;
  return GS_OK;
}

gs_status gs_set_densify_stats(gs_ctx* c, float* grad_accum, uint32_t* view_count) {
  if (!c) return GS_ERR_INVALID_ARG;
  if ((grad_accum == nullptr) != (view_count == nullptr))
    return fail(c, GS_ERR_INVALID_ARG, "grad_accum and view_count must both be set or both be NULL");
  if ((grad_accum && !aligned(grad_accum, 4)) || (view_count && !aligned(view_count, 4)))
    return fail(c, GS_ERR_INVALID_ARG, "statistics buffers must be 4-byte aligned");
  c->stat_accum = grad_accum;
  c->stat_count = view_count;
  return GS_OK;
}

gs_status gs_densify(gs_ctx* c, const gs_params* in, const gs_grads* m_in, const gs_grads* v_in,
                     const float* grad_accum, const uint32_t* view_count, const float* normals,
                     float grad_threshold, float scale_threshold, float min_opacity, const gs_grads* out,
                     const gs_grads* m_out, const gs_grads* v_out, int64_t out_n_pad, int64_t* n_out,
                     void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  gs_status s = check_params(c, in);
  if (s != GS_OK) return s;
  if (!m_in || !v_in || !out || !m_out || !v_out || !n_out)
    return fail(c, GS_ERR_INVALID_ARG, "moment, output and count pointers must be non-NULL");
  if (!(grad_threshold > 0.f) || !(scale_threshold > 0.f) || !(min_opacity > 0.f && min_opacity < 1.f) ||
      !std::isfinite(grad_threshold) || !std::isfinite(scale_threshold))
    return fail(c, GS_ERR_INVALID_ARG, "thresholds must be positive and min_opacity in (0, 1)");
  if (out_n_pad < 0) return fail(c, GS_ERR_INVALID_ARG, "out_n_pad must be >= 0");
  const gs_grads* sets[5] = {m_in, v_in, out, m_out, v_out};
  if (in->n > 0) {
    if (!grad_accum || !view_count || !normals) return fail(c, GS_ERR_INVALID_ARG, "statistics/normals NULL");
    for (const gs_grads* g : sets) {
      const float* q[5] = {g->means, g->log_scales, g->quats, g->opacity_logits, g->sh};
      for (const float* x : q)
        if (!x || !aligned(x, 4)) return fail(c, GS_ERR_INVALID_ARG, "a buffer pointer is NULL or misaligned");
    }
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  gs::DensifyArgs a;
  a.means = in->means;
  a.log_scales = in->log_scales;
  a.quats = in->quats;
  a.opacity_logits = in->opacity_logits;
  a.sh = in->sh;
  const float* mi[5] = {m_in->means, m_in->log_scales, m_in->quats, m_in->opacity_logits, m_in->sh};
  const float* vi[5] = {v_in->means, v_in->log_scales, v_in->quats, v_in->opacity_logits, v_in->sh};
  float* po[5] = {out->means, out->log_scales, out->quats, out->opacity_logits, out->sh};
  float* mo[5] = {m_out->means, m_out->log_scales, m_out->quats, m_out->opacity_logits, m_out->sh};
  float* vo[5] = {v_out->means, v_out->log_scales, v_out->quats, v_out->opacity_logits, v_out->sh};
  for (int k = 0; k < 5; ++k) {
    a.m[k] = mi[k];
    a.v[k] = vi[k];
    a.out_p[k] = po[k];
    a.out_m[k] = mo[k];
    a.out_v[k] = vo[k];
  }
  a.n = in->n;
  a.np_in = in->n_pad;
  a.sh_k = (in->sh_degree + 1) * (in->sh_degree + 1);
  a.grad_accum = grad_accum;
  a.view_count = view_count;
  a.normals = normals;
  a.grad_threshold = static_cast<double>(grad_threshold);
  a.log_scale_threshold = std::log(static_cast<double>(scale_threshold));
  a.logit_threshold = std::log(static_cast<double>(min_opacity) / (1.0 - static_cast<double>(min_opacity)));
  a.np_out = out_n_pad;
  a.block_counts = c->dens_counts;
  a.block_prefix = c->dens_prefix;
  a.totals = c->dens_totals;
  GS_CUDA(c, gs::launch_densify_count(a, st));
  GS_CUDA(c, cudaMemcpyAsync(c->dens_host, c->dens_totals, sizeof(uint4), cudaMemcpyDeviceToHost, st));
  GS_CUDA(c, cudaStreamSynchronize(st));
  const uint4 tot = *c->dens_host;
  const int64_t count = static_cast<int64_t>(tot.x) + tot.y + 2 * static_cast<int64_t>(tot.z);
  *n_out = count;
  if (count > out_n_pad)
    return fail(c, GS_ERR_CAPACITY, "densification gives %lld Gaussians; the output holds %lld",
                (long long)count, (long long)out_n_pad);
  GS_CUDA(c, gs::launch_densify_write(a, tot, st));
  return GS_OK;
}

gs_status gs_relocate(gs_ctx* c, const gs_grads* params, const gs_grads* m, const gs_grads* v, int64_t n,
                      int64_t n_pad, int32_t sh_degree, const float* normals, int64_t max_pairs,
                      float dead_opacity, float donor_opacity, int64_t* n_pairs, void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (!params || !m || !v || !n_pairs) return fail(c, GS_ERR_INVALID_ARG, "params, moments and n_pairs must be non-NULL");
  *n_pairs = 0;
  if (n < 0 || n_pad < n || n_pad % 4 != 0 || n > c->max_g)
    return fail(c, GS_ERR_INVALID_ARG, "n must be in [0, max_gaussians], n_pad >= n and a multiple of 4");
  if (sh_degree < 0 || sh_degree > 3) return fail(c, GS_ERR_INVALID_ARG, "sh_degree must be 0..3");
  if (max_pairs < 0 || (max_pairs > 0 && (!normals || !aligned(normals, 4))))
    return fail(c, GS_ERR_INVALID_ARG, "max_pairs must be >= 0 and normals non-NULL when it is > 0");
  if (!(dead_opacity > 0.f && dead_opacity < donor_opacity && donor_opacity < 1.f))
    return fail(c, GS_ERR_INVALID_ARG, "need 0 < dead_opacity < donor_opacity < 1");
  const gs_grads* sets[3] = {params, m, v};
  if (n > 0)
    for (const gs_grads* g : sets) {
      const float* q[5] = {g->means, g->log_scales, g->quats, g->opacity_logits, g->sh};
      for (const float* x : q)
        if (!x || !aligned(x, 4)) return fail(c, GS_ERR_INVALID_ARG, "a buffer pointer is NULL or misaligned");
    }
  if (n == 0 || max_pairs == 0) return GS_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!c->reloc_dead) GS_CUDA(c, cudaMalloc(reinterpret_cast<void**>(&c->reloc_dead), sizeof(uint32_t) * c->max_g));
  c->have_pre = c->have_fwd = false;  // the parameters change; so does the sort scratch
  gs::RelocateArgs a{};
  float* pp[5] = {params->means, params->log_scales, params->quats, params->opacity_logits, params->sh};
  float* mm[5] = {m->means, m->log_scales, m->quats, m->opacity_logits, m->sh};
  float* vv[5] = {v->means, v->log_scales, v->quats, v->opacity_logits, v->sh};
  for (int k = 0; k < 5; ++k) {
    a.p[k] = pp[k];
    a.m[k] = mm[k];
    a.v[k] = vv[k];
  }
  a.n = n;
  a.np = n_pad;
  a.sh_k = (sh_degree + 1) * (sh_degree + 1);
  const double dd = dead_opacity, dn = donor_opacity;
  a.dead_logit = std::log(dd / (1.0 - dd));
  a.donor_logit = std::log(dn / (1.0 - dn));
  a.block_counts = c->dens_counts;
  a.block_prefix = c->dens_prefix;
  a.totals = c->dens_totals;
  a.dead = c->reloc_dead;
  a.donor_keys = c->dkeys[0];
  a.donor_vals = c->dvals[0];
  a.err = &c->info_dev->device_error;
  GS_CUDA(c, gs::launch_relocate_classify(a, st));
  GS_CUDA(c, cudaMemcpyAsync(c->dens_host, c->dens_totals, sizeof(uint4), cudaMemcpyDeviceToHost, st));
  GS_CUDA(c, cudaStreamSynchronize(st));
  const int64_t dead = c->dens_host->x, donors = c->dens_host->y;
  const int64_t pairs = std::min(std::min(dead, donors), max_pairs);
  *n_pairs = pairs;
  if (pairs == 0) return GS_OK;
  // donors by descending size, stably (ties stay in index order)
  gs::SortBuffers b;
  b.keys[0] = c->dkeys[0];
  b.keys[1] = c->dkeys[1];
  b.vals[0] = c->dvals[0];
  b.vals[1] = c->dvals[1];
  b.hist = c->hist;
  b.offsets = c->offsets;
  b.chunk_counts = c->chunk_counts;
  b.err = &c->info_dev->device_error;
  gs::SortPlan plan;
  plan.n = donors;
  plan.key_bits = 32;
  plan.passes = 4;
  plan.tiles = (donors + gs::kSortTileKeys - 1) / gs::kSortTileKeys;
  int sorted = 0;
  GS_CUDA(c, gs::launch_sort(plan, b, &sorted, st));
  a.sorted_donors = c->dvals[sorted];
  a.normals = normals;
  a.pairs = pairs;
  GS_CUDA(c, gs::launch_relocate_pairs(a, st));
  return GS_OK;
}

gs_status gs_opacity_reset(float* logits, float* m, float* v, int64_t n, float max_opacity, void* stream) {
  if (n < 0 || !(max_opacity > 0.f && max_opacity < 1.f)) return GS_ERR_INVALID_ARG;
  if (n > 0 && (!logits || !m || !v)) return GS_ERR_INVALID_ARG;
  const double mo = static_cast<double>(max_opacity);
  const float cap = static_cast<float>(std::log(mo / (1.0 - mo)));
  cudaError_t e = gs::launch_opacity_reset(logits, m, v, n, cap, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}


gs_status gs_loss_charbonnier(gs_ctx* c, const float* image, const float* target, int32_t height,
                              int32_t width, const float* gain, const float* bias, float delta,
                              double* out, float* dloss_dimage, void* stream) {
  if (!c) return GS_ERR_INVALID_ARG;
  if (height <= 0 || width <= 0 || height > c->max_h || width > c->max_w)
    return fail(c, GS_ERR_INVALID_ARG, "image %dx%d outside the context's maximum", width, height);
  if (!image || !target || !out || !gain || !bias || !aligned(image, 4) || !aligned(target, 4) ||
      !aligned(out, 8) || (dloss_dimage && !aligned(dloss_dimage, 4)))
    return fail(c, GS_ERR_INVALID_ARG, "loss pointers must be non-NULL and aligned");
  if (!(delta > 0.f) || !std::isfinite(delta)) return fail(c, GS_ERR_INVALID_ARG, "delta must be positive");
  for (int k = 0; k < 3; ++k)
    if (!std::isfinite(gain[k]) || !std::isfinite(bias[k]))
      return fail(c, GS_ERR_INVALID_ARG, "gain and bias must be finite");
  gs::CharbonnierArgs a;
  a.x = image;
  a.y = target;
  a.pixels = static_cast<int64_t>(height) * width;
  for (int k = 0; k < 3; ++k) {
    a.gain[k] = gain[k];
    a.bias[k] = bias[k];
  }
  a.delta = delta;
  a.dx = dloss_dimage;
  a.partials = c->charb_partials;
  a.counter = c->charb_counter;
  a.out = out;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prof_begin(c, st);
  GS_CUDA(c, gs::launch_charbonnier(a, st));
  prof_end(c, GS_STAGE_LOSS, a.pixels, st);
  return GS_OK;
}

}  // extern "C"
