/*
 * gs_api.h - C ABI of the B200 (sm_100a) differentiable tile-based
 * Gaussian-splat rasteriser: preprocess, tile sort + forward blend, fused
 * L1 + D-SSIM loss, blend + projection backward, and a fused Adam step; plus
 * the training loop's other steps on the same data: the Charbonnier +
 * exposure loss, camera-pose gradients, adaptive density control and the
 * recycling of dead Gaussians, and the data-parallel gradient exchange fused
 * with Adam over peer memory.
 *
 * Conventions shared by every call
 *   - Every data pointer is a DEVICE pointer owned by the caller, unless the
 *     argument says "host". Buffers are never freed or retained by the library
 *     beyond the call, except the scratch a gs_ctx owns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Work is enqueued asynchronously on it. gs_render_forward is the one call
 *     that waits on the stream (it reads the entry count back to the host).
 *     The training step's kernels are launched with programmatic dependent
 *     launch: a kernel may be scheduled while the work ahead of it on the
 *     stream drains, but it touches no memory before that work has completed,
 *     so stream order holds as for ordinary launches.
 *   - Parameters are structure-of-arrays, planar float32, with n <= n_pad,
 *     n_pad a multiple of 4 and 16-byte aligned base pointers, so every plane
 *     starts 16-byte aligned:
 *         means           [3][n_pad]
 *         log_scales      [3][n_pad]
 *         quats           [4][n_pad]      (w, x, y, z), any non-zero length
 *         opacity_logits  [n_pad]
 *         sh              [3][(sh_degree+1)^2][n_pad]   k = 0 is the base RGB
 *     Entries n .. n_pad-1 are ignored by the rasteriser (Adam still updates
 *     them as ordinary scalars; with zero gradient they do not move).
 *   - Images are [3][height][width] float32 (channel-major, row-major);
 *     per-pixel maps are [height][width].
 *   - Pixel (i, j) sits at continuous coordinate (i, j). Camera axes: x right,
 *     y down, z forward; p_cam = R p_world + t.
 *   - Every call returns a gs_status. Argument and size errors are detected on
 *     the host before anything is enqueued (GS_ERR_INVALID_ARG). A failed CUDA
 *     launch returns GS_ERR_CUDA. A fault recorded by a kernel's own bounded
 *     checks returns GS_ERR_DEVICE. No kernel traps or waits without bound.
 *     gs_last_error() gives a one-line description of the last failure.
 *
 * Citations name the web pages this method is described on:
 *   [DR]  "Differentiable rasterisation" (splat-report.pages.dev).
 *   [TBR] "Tile-based differentiable rasterization in 3DGS"
 *         (learn-ml-visualized-interactive).
 *   [SN]  Gaussian splatting training study notes (bailiping.com).
 *   [GS]  "How a computer rebuilds a real place out of soft colored dots
 *         called Gaussian Splats" (taosengine.com).
 */
#ifndef GS_API_H
#define GS_API_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GS_OK = 0,
  GS_ERR_INVALID_ARG = 1, /* bad pointer, size, order of calls or capacity request */
  GS_ERR_CAPACITY = 2,    /* more (Gaussian, tile) entries than the context holds */
  GS_ERR_CUDA = 3,        /* a CUDA API call or kernel launch failed */
  GS_ERR_DEVICE = 4       /* a kernel's bounded self-check recorded a fault */
} gs_status;

/* Pinhole camera (host struct, passed by pointer, copied by value). */
typedef struct {
  int32_t width, height;
  float fx, fy, cx, cy;
  float R[9];      /* world -> camera rotation, row-major */
  float t[3];      /* p_cam = R p_world + t */
  float campos[3]; /* camera centre in world space; origin of the view direction */
  float bg[3];     /* background colour */
  float near_z;    /* Gaussians with camera depth <= near_z are culled */
} gs_camera;

/* Read-only parameters (host struct holding device pointers). */
typedef struct {
  const float *means, *log_scales, *quats, *opacity_logits, *sh;
  int64_t n, n_pad;
  int32_t sh_degree;     /* storage degree, 0..3 */
  int32_t active_degree; /* bands used for colour, 0..sh_degree */
} gs_params;

/* Parameter gradients, same layout as gs_params. gs_render_backward ADDS
 * into them (several views may be accumulated); gs_adam_step zeroes them. */
typedef struct {
  float *means, *log_scales, *quats, *opacity_logits, *sh;
} gs_grads;

/* Opaque context. It owns the scratch of one camera in flight: per-Gaussian
 * screen state, sort keys and values (double-buffered), per-tile ranges,
 * per-Gaussian screen-space gradients and the loss partial sums. */
typedef struct gs_ctx gs_ctx;

/* Allocates a context for up to max_gaussians Gaussians, max_entries
 * (Gaussian, tile) entries and images up to max_width x max_height. Device
 * memory: about 150 B per Gaussian plus 80 B per entry (sort buffers and the
 * blend's per-warp lists of the entries that blend in each 8x4 pixel block).
 * The entry budget mirrors the global (blob, tile) budget of [GS] section
 * "Why tiling, and the five stages". The caller owns *ctx and frees it with
 * gs_destroy. Returns GS_ERR_INVALID_ARG for non-positive sizes and
 * GS_ERR_CUDA if device memory cannot be allocated (nothing is leaked). */
gs_status gs_create(gs_ctx **ctx, int64_t max_gaussians, int64_t max_entries,
                    int32_t max_width, int32_t max_height);
void gs_destroy(gs_ctx *ctx);
/* Human-readable description of the last failure on this context ("" if none).
 * The string is owned by the context. */
const char *gs_last_error(const gs_ctx *ctx);

/* Context options. */
typedef enum {
  /* Value 1: each Gaussian's tile rect uses the opacity-aware radius of [GS]
   * section "Why tiling, and the five stages" (the code after the list):
   * r = sqrt(2 E) sqrt(lambda_max) with E = min(4.5, ln(max(255 o, 1.0001))),
   * alpha_min = 1/255, instead of 3 sqrt(lambda_max); o is the opacity times
   * the compensation factor when GS_OPTION_MIP_COMPENSATION is set. Alpha
   * stays below 1/255 in every tile it drops, so the image and gradients do
   * not change; the (Gaussian, tile) lists get shorter. Value 0 (the
   * default): the 3-sigma rect. */
  GS_OPTION_OPACITY_RECT = 1,
  /* Value 1: the backward accumulates each Gaussian's screen-space gradient
   * sums as 64-bit integers in 2^-40 fixed point instead of float32 atomics
   * (the integer-atomic idea of [GS] section "Making the parallel sums exact:
   * fixed-point, and the conic trick", with a 64-bit word and a finer scale
   * instead of 32 bits x 16384, because mean-reduced losses give per-pixel
   * gradients near 1e-7). Integer sums do not depend on the order of the
   * additions, so gs_render_backward and gs_render_backward_adam are then
   * bitwise reproducible. Enabling it allocates 72 B per Gaussian of the
   * context (GS_ERR_CUDA if that fails). Value 0 (the default): float32
   * atomics. */
  GS_OPTION_DETERMINISTIC = 2,
  /* Value 1: each Gaussian's opacity is multiplied by the Mip-Splatting
   * compensation factor that [GS] section "Flattening a 3D blob into a 2D
   * oval (EWA projection)" names (alpha = min(0.99, opacity * comp *
   * exp(-e)) in "The painting itself", and opacity * comp in the
   * opacity-aware radius), with the factor of Mip-Splatting's 2D filter,
   * comp = sqrt(det V / det(V + 0.3 I)) for the screen covariance V before
   * the 0.3 px^2 dilation (0 if det V <= 0): the dilated splat keeps the
   * integrated weight of the undilated one. The backward carries its
   * gradient into the covariance (the pages' "comp" slot). Value 0 (the
   * default): no factor. */
  GS_OPTION_MIP_COMPENSATION = 3
} gs_option;

/* Sets a context option; it applies from the next gs_preprocess (the state
 * of the camera in flight is discarded). Errors: GS_ERR_INVALID_ARG for an
 * unknown option or value. */
gs_status gs_set_option(gs_ctx *ctx, int32_t option, int32_t value);

/* Step 1 - preprocess, one thread per Gaussian ([SN] slides on the
 * parametrisation and "J is the 2 x 3 Jacobian of perspective projection";
 * [GS] sections "Flattening a 3D blob into a 2D oval (EWA projection)" and
 * "Spherical harmonics: color that changes with viewing angle"):
 * p_c = R p + t; cull if Z <= near_z; Sigma = R(q/|q|) S S^T R^T with
 * S = diag(exp(log_scales)); Sigma' = J W Sigma W^T J^T + 0.3 I with
 * J = [fx/Z, 0, -fx X/Z^2; 0, fy/Z, -fy Y/Z^2]; conic = Sigma'^-1; mean2d;
 * radius 3 sqrt(lambda_max(Sigma')); rect of the 16x16 tiles meeting
 * mean2d +- radius; opacity = sigmoid(logit); colour = max(0, sum_k sh_k Y_k(v))
 * at v = normalize(p - campos) using bands up to active_degree.
 * The geometry is evaluated in float64 (depth key = float32(Z)), the colour in
 * float32. Results stay in the context for gs_render_forward/backward.
 * Errors: GS_ERR_INVALID_ARG if n > max_gaussians, n_pad < n, n_pad % 4 != 0,
 * a degree is out of range, a pointer is NULL or misaligned, or the camera is
 * larger than the context's maximum image. */
gs_status gs_preprocess(gs_ctx *ctx, const gs_params *params, const gs_camera *cam, void *stream);

/* Step 2 - tile lists and forward blend ([GS] sections "Why tiling, and the
 * five stages" and "The painting itself: front-to-back alpha compositing";
 * [DR] section "The trick: recompute the blend state instead of storing it";
 * [SN] slide on alpha and the background term).
 * Orders the (Gaussian, tile) entries by (tile, depth, index): the visible
 * Gaussians are sorted by depth with a stable LSD radix sort, one
 * entry per touched tile is emitted in that order (prefix sum over
 * tiles_touched), and the entries are sorted stably by tile; then per-tile
 * ranges are extracted and each 16x16 tile is blended front to back:
 * alpha = min(0.99, o exp(-e)), e = 1/2 (A dx^2 + C dy^2) + B dx dy, entries
 * with alpha < 1/255 skipped, C += T alpha c, T *= 1 - alpha, and the walk
 * stops after the entry that takes T below 1e-4. Writes
 * image_chw = C + T bg, final_T = T, and n_contrib = 1 + list position of the
 * last blended entry (0 if none). *num_entries_out (HOST pointer, may be
 * NULL) receives the entry count. This call synchronises `stream` once to
 * read the entry count. Errors: GS_ERR_INVALID_ARG if gs_preprocess has not
 * run for this camera size; GS_ERR_CAPACITY (nothing written) if the entry
 * count exceeds max_entries. */
gs_status gs_render_forward(gs_ctx *ctx, const gs_camera *cam, float *image_chw, float *final_T,
                            int32_t *n_contrib, int64_t *num_entries_out, void *stream);

/* Step 3 - fused photometric loss ([SN] slides "An iteration samples a camera
 * and differentiates its image loss", L1, and "11 x 11 Gaussian window,
 * standard deviation 1.5 pixels"): L = (1 - lambda) L1 + lambda (1 - SSIM),
 * L1 = mean |x - y| over 3HW, SSIM = mean over 3HW of the SSIM map with an
 * 11x11 Gaussian window (sigma 1.5), C1 = 0.01^2, C2 = 0.03^2 and zero padding.
 * Writes loss_out[0..2] = {L, L1, SSIM} (DEVICE pointer to 3 doubles; the
 * reduction is deterministic) and, if dloss_dimage is not NULL, dL/dx with the
 * L1 subgradient 0 at a zero residual. Works on any image up to the context's
 * maximum size. Errors: GS_ERR_INVALID_ARG for bad sizes or pointers. */
gs_status gs_loss_l1_dssim(gs_ctx *ctx, const float *image_chw, const float *target_chw,
                           int32_t height, int32_t width, float lambda, double *loss_out,
                           float *dloss_dimage, void *stream);

/* Step 4 - backward ([DR] sections "The trick" and "From a pixel error back to
 * a quaternion"; [GS] sections "The clever bit: a single backward sweep through
 * the blend", "From a pixel's blame to the oval's shape and place", "The
 * covariance chain", "Where the position gradient comes from"; [SN] slide
 * "r is the RGB loss gradient"). Re-walks each tile back to front from each
 * pixel's last contributor, recovering T by division by (1 - alpha), reduces
 * the per-Gaussian screen gradients within each warp before the global
 * atomics, then chains them through conic, Sigma', J, W, quaternion/scale,
 * opacity and SH (including the view-direction path into the means).
 * ADDS the result into *grads. `params` and `cam` must be the ones given to
 * the last gs_preprocess, and final_T / n_contrib the outputs of the last
 * gs_render_forward. Errors: GS_ERR_INVALID_ARG if the forward has not run
 * or the inputs do not match it. Gradients are not bitwise reproducible
 * (float32 atomics) unless GS_OPTION_DETERMINISTIC is set. */
gs_status gs_render_backward(gs_ctx *ctx, const gs_params *params, const gs_camera *cam,
                             const float *final_T, const int32_t *n_contrib,
                             const float *dloss_dimage, gs_grads *grads, void *stream);

/* Step 3 without allocation - the same fused loss as gs_loss_l1_dssim, for
 * callers that cannot allocate device memory where they need the loss: a
 * host application whose own allocator owns the GPU's memory and hands the
 * library only input and output pointers, and real-time loops whose memory is
 * fixed after start-up (cudaMalloc can synchronise the device and stall the
 * loop). The paper has no counterpart; this is an interface convenience of
 * this library.
 * It needs no context: the kernel's scratch (per-CTA partial sums and a
 * completion counter, about 0.2 MB) is a file-scope __device__ array that
 * every GPU loading the library holds until the process exits. The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current), so make that first call before any stream
 * capture. All calls on a device share the one array: calls that overlap on
 * the GPU (other streams, other threads) race and must be serialised by the
 * caller. Arguments and outputs as gs_loss_l1_dssim. Returns
 * GS_ERR_CAPACITY, with nothing enqueued, for an image wider or taller than
 * 4096 pixels; GS_ERR_INVALID_ARG for bad pointers or sizes; GS_ERR_CUDA if
 * the symbol lookup, the counter reset or the launch fails. Allocates
 * nothing and frees nothing. */
gs_status gs_loss_l1_dssim_noalloc(const float *image_chw, const float *target_chw, int32_t height,
                                   int32_t width, float lambda, double *loss_out,
                                   float *dloss_dimage, void *stream);

/* Steps 4 + 5 in one pass - the backward of gs_render_backward followed, in the
 * same pass over the parameters, by the Adam step of gs_adam_step on every
 * group: for each scalar g = grads + this view's gradient, then the Adam update
 * with that group's learning rate; params are updated IN PLACE (the pointers in
 * *params must be writable), m and v are updated, and grads are left zeroed.
 * The result is bit-identical to gs_render_backward(..., grads) followed by
 * gs_adam_step on each group, but the gradient makes no separate round trip
 * through memory ([DR] section "From a pixel error back to a quaternion":
 * every group updated by Adam with its own learning rate). lr is a HOST array
 * of 5 learning rates in the order means, log_scales, quats, opacity_logits,
 * sh; exp_avg and exp_avg_sq hold the first and second moments in the
 * parameter layout. grads may be NULL when there is no accumulated gradient
 * (one view per step, as in the method's training loop): the update then uses
 * this view's gradient alone and no gradient buffer is read or written, which
 * saves 8 of the 32 bytes each scalar moves; the result equals the call with
 * an all-zero grads buffer. Errors as gs_render_backward, plus
 * GS_ERR_INVALID_ARG for a NULL moment pointer, step < 1 or betas outside
 * [0, 1). */
gs_status gs_render_backward_adam(gs_ctx *ctx, const gs_params *params, const gs_camera *cam,
                                  const float *final_T, const int32_t *n_contrib,
                                  const float *dloss_dimage, gs_grads *grads, gs_grads *exp_avg,
                                  gs_grads *exp_avg_sq, const float *lr, float beta1, float beta2,
                                  float eps, int32_t step, void *stream);

/* Step 5 - fused Adam over one flat float32 buffer of `count` scalars
 * ([GS] Adam paragraph after "Proving the blame is right"; [DR] per-group
 * learning rates): m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
 * p -= lr (m / (1 - b1^step)) / (sqrt(v / (1 - b2^step)) + eps); g = 0.
 * step >= 1. Call once per parameter group to give each its own lr.
 * Errors: GS_ERR_INVALID_ARG for NULL pointers, count < 0 or step < 1. */
gs_status gs_adam_step(float *param, float *grad, float *m, float *v, int64_t count, float lr,
                       float beta1, float beta2, float eps, int32_t step, void *stream);

/* ------------------------------------------- data-parallel training ------
 * Several GPUs of one node train one set of Gaussians, each rendering its own
 * camera of the iteration ([GS] "Per step": one photo per step; with R
 * ranks the batch gradient is the mean of the R per-rank gradients). Each
 * rank owns a contiguous shard of the flat parameter buffer, the only part
 * whose Adam moments it keeps.
 *
 * Step 5, data-parallel form - the gradient exchange fused with Adam over
 * one rank's shard (one parameter group's part of it, so each group keeps its
 * own lr): g = grad_scale * (grads[0][i] + ... + grads[n_grads-1][i]) summed
 * in that order (bitwise the same on every run), then the gs_adam_step update
 * of param[i], m[i], v[i] with g, then param[i] is also stored to every
 * param_copies[d][i]. With zero_grads != 0 every gradient source is zeroed
 * after it is read (so n_grads = 1, grad_scale = 1, zero_grads = 1 is
 * gs_adam_step, bit for bit). grads and param_copies are HOST arrays of
 * DEVICE pointers, each at the shard's first scalar: this GPU's own memory,
 * or a peer GPU's memory opened with gs_shared_open (read and written with
 * plain loads and stores over NVLink; no multicast). 1 <= n_grads <= 8,
 * 0 <= n_copies <= 8. The caller orders the call after every rank's
 * gradient is complete and every rank's next use of its parameters after
 * every rank's call (stream-ordered barriers); the kernel itself waits on
 * nothing. float4 accesses when every pointer is 16-byte aligned and count is
 * a multiple of 4. Errors: GS_ERR_INVALID_ARG for NULL or misaligned
 * (4-byte) pointers, counts out of range, count < 0, step < 1, bad betas or
 * a non-finite lr or grad_scale; GS_ERR_CUDA if the launch fails. */
gs_status gs_adam_step_reduce(float *param, float *m, float *v, int64_t count, float *const *grads,
                              int32_t n_grads, float *const *param_copies, int32_t n_copies,
                              int32_t zero_grads, float grad_scale, float lr, float beta1, float beta2,
                              float eps, int32_t step, void *stream);

/* ------------------------------------- data-parallel update from views --
 * The alternative to exchanging parameter gradients: each rank runs only the
 * blend backward of its camera, and the rank that owns a range of Gaussians
 * reads every rank's view of them (about 100 B per Gaussian and view instead
 * of a 236 B gradient), runs the projection backward of every view, averages
 * and applies Adam in one pass ([GS] section "Per step": one photo per step;
 * with one photo per rank the batch gradient is the mean of the ranks'
 * gradients). */

/* One rank's view of the Gaussians after gs_render_backward_screen: DEVICE
 * pointers (this GPU's, or a peer's opened with gs_shared_open) to its
 * per-Gaussian screen records, raw screen-gradient sums, touched counts, clamp
 * flags and its camera record. Each is the start of a device allocation of
 * the context, so gs_shared_handle can make an IPC handle for it. */
typedef struct {
  const void *screen;
  const float *sums;
  const uint32_t *touched;
  const uint8_t *clamped;
  const void *camera;
} gs_view;

/* The blend backward of the last forward alone (step 4 up to the raw screen
 * sums; [GS] "The clever bit: a single backward sweep through the blend"):
 * the sums, the screen records, the flags and the camera stay in the context
 * as its view, for gs_adam_step_views on this or other ranks. Arguments and
 * errors as gs_render_backward. Density statistics are not accumulated. */
gs_status gs_render_backward_screen(gs_ctx *ctx, const gs_params *params, const gs_camera *cam,
                                    const float *final_T, const int32_t *n_contrib,
                                    const float *dloss_dimage, void *stream);

/* The context's view buffers (valid for the whole life of the context; their
 * contents are those of the last gs_render_backward_screen). */
gs_status gs_get_view(const gs_ctx *ctx, gs_view *out);

/* The IPC handle (GS_SHARED_HANDLE_BYTES bytes, written to the HOST array
 * `handle`) of a device allocation that starts at ptr, for gs_shared_open on
 * another rank. GS_ERR_CUDA if ptr is not the start of a device allocation. */
gs_status gs_shared_handle(const void *ptr, unsigned char *handle);

/* Steps 4 (projection part) + 5 for the Gaussians [g_lo, g_hi) of this rank,
 * over n_views ranks' views (1..8, in rank order): per Gaussian, the
 * projection backward of every view that touched it, summed in rank order and
 * multiplied by grad_scale (1 / ranks for the batch mean), then the Adam step
 * of each scalar with its group's learning rate (lr: HOST array of 5, group
 * order means, log_scales, quats, opacity_logits, sh). The parameters in
 * *params are updated IN PLACE and also written into each of the n_copies
 * (0..8) other ranks' parameter buffers (group pointers, usually peer memory;
 * plain stores, no multicast). The result equals gs_render_backward on each
 * view, gradients summed in rank order, then gs_adam_step_reduce with the same
 * grad_scale, up to float32 rounding (the same operations in another kernel),
 * and every rank's parameters end bit-identical. Only this rank's moments of
 * [g_lo, g_hi) are read and written. g_lo and g_hi are multiples of 4 within
 * [0, n_pad]; parameters, moments and copies 16-byte aligned; every view's
 * parameters must equal these (the ranks hold replicas). The caller orders the
 * call after every rank's gs_render_backward_screen and every rank's next
 * forward after every rank's call (stream-ordered barriers); the kernel waits
 * on nothing. Errors: GS_ERR_INVALID_ARG for NULL or misaligned pointers,
 * counts or ranges out of bounds, step < 1, bad betas or non-finite lr /
 * grad_scale; GS_ERR_CUDA if the launch fails. */
gs_status gs_adam_step_views(gs_ctx *ctx, const gs_params *params, const gs_view *views, int32_t n_views,
                             int64_t g_lo, int64_t g_hi, const gs_grads *copies, int32_t n_copies,
                             gs_grads *exp_avg, gs_grads *exp_avg_sq, const float *lr, float grad_scale,
                             float beta1, float beta2, float eps, int32_t step, void *stream);

/* Device memory that other processes on the node can map (CUDA IPC): the
 * buffers whose shards gs_adam_step_reduce reads and writes on peers.
 * gs_shared_alloc allocates `bytes` on the current device, zero-filled, and
 * writes its GS_SHARED_HANDLE_BYTES-byte handle to the HOST array `handle`
 * (to be sent to the other ranks); the caller frees it with gs_shared_free.
 * gs_shared_open maps another process's allocation from its handle (peer
 * access enabled lazily) and gs_shared_close unmaps it. Handles cannot be
 * opened by the process that made them. Errors: GS_ERR_INVALID_ARG for NULL
 * arguments or bytes <= 0; GS_ERR_CUDA if the CUDA call fails (nothing is
 * leaked, *ptr is NULL). */
#define GS_SHARED_HANDLE_BYTES 64
gs_status gs_shared_alloc(int64_t bytes, void **ptr, unsigned char *handle);
gs_status gs_shared_open(const unsigned char *handle, void **ptr);
gs_status gs_shared_close(void *ptr);
gs_status gs_shared_free(void *ptr);

/* ------------------------------------------------------------ profiling --
 * gs_profile_enable takes a set of flags (0 turns profiling off):
 *   GS_PROFILE_TIME  - every kernel launch a context makes is bracketed by
 *                      CUDA events on the call's stream (a few microseconds
 *                      of host time per launch; leave it off for throughput
 *                      runs). The kernels timed are the ones a run without
 *                      profiling launches.
 *   GS_PROFILE_COUNT - the two blends count (pixel, Gaussian) pairs: their
 *                      counting variants run instead (slower, so stage times
 *                      taken together with this flag are those variants').
 * gs_profile_read waits for the recorded events, returns per-stage totals
 * accumulated since the previous read and resets them. Each output is a HOST
 * array of GS_NUM_STAGES entries (any may be NULL): ms = summed kernel time,
 * launches = kernel launches, work = the units processed (Gaussians for the
 * per-Gaussian stages - n_pad for the fused backward + Adam pass -, visible
 * Gaussians x passes for the depth sort, entries x passes for the tile sort,
 * entries for the duplication and ranges, pixels for the loss; for the two
 * blends, when counting, the (pixel, Gaussian) pairs the method's walk
 * visits: every list entry up to the pixel's stopping point in the forward,
 * every entry before its last contributor in the backward, and 0 when not
 * counting), blended = for the two blends the pairs that actually blend
 * (alpha >= 1/255 before the walk stops) when counting, 0 elsewhere.
 * Unknown flags give GS_ERR_INVALID_ARG. gs_adam_step takes no context and is
 * not profiled here. */
typedef enum { GS_PROFILE_TIME = 1, GS_PROFILE_COUNT = 2 } gs_profile_flag;
typedef enum {
  GS_STAGE_PREPROCESS = 0,
  GS_STAGE_SCAN = 1,
  GS_STAGE_DUPLICATE = 2,
  GS_STAGE_SORT = 3,
  GS_STAGE_RANGES = 4,
  GS_STAGE_BLEND_FORWARD = 5,
  GS_STAGE_LOSS = 6,
  GS_STAGE_BLEND_BACKWARD = 7,
  GS_STAGE_PREPROCESS_BACKWARD = 8,
  GS_STAGE_BACKWARD_ADAM = 9, /* the fused projection backward + Adam pass */
  GS_STAGE_DEPTH_SORT = 10,   /* compaction + depth sort of the visible Gaussians */
  GS_STAGE_CAMERA_BACKWARD = 11, /* camera-pose gradient (when gs_set_camera_grad is on) */
  GS_STAGE_VIEWS_ADAM = 12,      /* data-parallel update from the views' screen sums */
  GS_NUM_STAGES = 13
} gs_stage;

gs_status gs_profile_enable(gs_ctx *ctx, int32_t enabled);
gs_status gs_profile_read(gs_ctx *ctx, double *ms, int64_t *launches, int64_t *work,
                          int64_t *blended);
/* Static name of a stage ("preprocess", "sort", ...), or "" if out of range. */
const char *gs_stage_name(int32_t stage);

/* ---------------------------------------------------------------- debug --
 * Copies of the context's internal state for stage-by-stage checks. Each
 * output is a DEVICE pointer and may be NULL. Copies are asynchronous on
 * `stream`. */

/* After gs_preprocess, for the n Gaussians: mean2d [n][2], conic [n][3]
 * (A, B, C), opacity [n], rgb [n][3], depth [n] (float32 camera Z),
 * rect [n][4] (x0, y0, x1, y1 inclusive tile indices; x0 > x1 when culled),
 * tiles_touched [n], clamped [n] (bit c set when colour channel c was
 * clamped at 0). */
gs_status gs_debug_preprocess(gs_ctx *ctx, float *mean2d, float *conic, float *opacity,
                              float *rgb, float *depth, int32_t *rect, int32_t *tiles_touched,
                              uint8_t *clamped, void *stream);
/* After gs_render_forward: the sorted Gaussian index per entry [K], the tile
 * per entry [K], and per-tile [lo, hi) ranges [tiles_y * tiles_x][2]. */
gs_status gs_debug_sorted(gs_ctx *ctx, int32_t *ids, int32_t *tiles, int32_t *ranges,
                          void *stream);
/* After gs_render_backward: per-Gaussian screen-space gradient [n][9] =
 * dL/d(mean2d x, mean2d y, A, B, C, opacity, r, g, b). */
gs_status gs_debug_screen_grads(gs_ctx *ctx, float *out, void *stream);

/* Step 3, second loss ([GS] the loss paragraph before "The chain rule, in one
 * breath"): a Charbonnier loss with a per-photo exposure correction,
 * err = gain_c C + bias_c - target per channel c, root = sqrt(err^2 +
 * delta^2), pixel loss = sum_c root - 3 delta (the page uses delta = 0.03),
 * image loss = the mean over the H W pixels. image_chw and target_chw are
 * [3][H][W] DEVICE float32; gain and bias are HOST arrays of 3. out is a
 * DEVICE array of 7 doubles: {loss, dL/dgain[3], dL/dbias[3]};
 * dloss_dimage (DEVICE [3][H][W], may be NULL) receives gain_c err / root / (H W).
 * The reductions are float64 in a fixed order (deterministic). Errors:
 * GS_ERR_INVALID_ARG for bad pointers, an image larger than the context's
 * maximum, delta <= 0 or non-finite gain / bias. */
gs_status gs_loss_charbonnier(gs_ctx *ctx, const float *image_chw, const float *target_chw,
                              int32_t height, int32_t width, const float *gain, const float *bias,
                              float delta, double *out, float *dloss_dimage, void *stream);

/* ------------------------------------------------------ density control --
 * Adaptive density control, run between training steps ([SN] slides "Where
 * to add capacity" and "A separate heuristic": the screen-space centre
 * gradient magnitude averaged over the views that saw a Gaussian flags
 * regions to densify; small flagged Gaussians are cloned, large ones split;
 * very low opacity prunes; opacity reset clamps opacity to at most 0.01;
 * [GS] "Densification": split halves shrink by 1.6 and restart their Adam
 * moments). The thresholds are the caller's settings, as the pages say. */

/* Registers two DEVICE buffers of max_gaussians entries that every later
 * gs_render_backward / gs_render_backward_adam on this context accumulates
 * into: grad_accum[i] += |dL/dmean2d_i| (Euclidean norm, pixels) and
 * view_count[i] += 1 for every Gaussian the view touched (tiles_touched > 0).
 * The caller zeroes them when it starts a statistics window. Pass NULL for
 * both to stop accumulating. Errors: GS_ERR_INVALID_ARG if exactly one is
 * NULL. */
gs_status gs_set_densify_stats(gs_ctx *ctx, float *grad_accum, uint32_t *view_count);

/* Camera-pose gradient ([GS] "Forgiving the camera and the light": the render
 * depends on the camera, so backprop gives it a gradient, which a trainer
 * uses to refine imperfect poses). With out set (a DEVICE array of 6 doubles,
 * 8-byte aligned), every later gs_render_backward / gs_render_backward_adam
 * also writes to out the gradient of the loss with respect to this view's
 * pose, for the update R <- exp([w]x) R, t <- t + dt of the camera given to
 * the call: out = {dL/dw_x, dL/dw_y, dL/dw_z, dL/dt_x, dL/dt_y, dL/dt_z}
 * (overwritten, not accumulated: each photo has its own pose). It is the
 * exact derivative: the position path of that section's code, plus the
 * rotation of each camera-space covariance and the move of the camera centre
 * -R^T t in the colours' view directions. It is computed from the parameters
 * passed to the call, before the fused call updates them. It is summed in
 * float64 in a fixed order (deterministic for a given screen gradient, so
 * bitwise reproducible with GS_OPTION_DETERMINISTIC). out = NULL turns it off
 * (the default). The context keeps the pointer; the caller keeps the buffer
 * alive. Errors: GS_ERR_INVALID_ARG for a NULL ctx or a misaligned out. */
gs_status gs_set_camera_grad(gs_ctx *ctx, double *out);

/* One densification pass from the set `in` (n Gaussians, planar with
 * in->n_pad) to the set `out` (planar with stride out_n_pad, written through
 * the float pointers of a gs_grads), moments m/v alongside. For Gaussian i,
 * with avg = grad_accum[i] / view_count[i] (float64), s_max = the largest
 * log-scale and o = sigmoid(logit):
 *   prune  if logit < logit(min_opacity)                 -> not written;
 *   else if view_count[i] > 0 and avg >= grad_threshold:
 *     clone if s_max <= log(scale_threshold)            -> i kept + one copy,
 *     split otherwise                                   -> i replaced by two
 *       children: mean + R(q/|q|) diag(exp(log-scales)) z_k with the caller's
 *       N(0, 1) draws z_k = normals[i][k][0..2] (k = 0, 1), log-scales
 *       - ln(1.6), the other parameters copied;
 *   else kept.
 * Output order: the kept Gaussians (cloned parents included) in index order,
 * then the clones in parent order, then the split children (child 0, child 1)
 * in parent order. Kept Gaussians keep their moments; clones and children
 * start at zero. *n_out (HOST) receives the new count; entries beyond it are
 * not written. The comparisons are taken in float64 against thresholds
 * converted once on the host, so they are exact. This call synchronises
 * `stream` once (to read the count). Errors: GS_ERR_INVALID_ARG for bad
 * pointers, n > the context's max_gaussians, a non-positive threshold or
 * min_opacity outside (0, 1); GS_ERR_CAPACITY (nothing written) if the new
 * count exceeds out_n_pad. */
gs_status gs_densify(gs_ctx *ctx, const gs_params *in, const gs_grads *m_in, const gs_grads *v_in,
                     const float *grad_accum, const uint32_t *view_count, const float *normals,
                     float grad_threshold, float scale_threshold, float min_opacity,
                     const gs_grads *out, const gs_grads *m_out, const gs_grads *v_out,
                     int64_t out_n_pad, int64_t *n_out, void *stream);

/* Opacity reset over n Gaussians: logit = min(logit, logit(max_opacity)) and
 * the Adam moments of the opacity logits set to zero ([SN] "A separate
 * heuristic": reset clamps opacity down to at most 0.01, the usual
 * max_opacity). All pointers DEVICE, [n] floats. Errors: GS_ERR_INVALID_ARG
 * for NULL pointers, n < 0 or max_opacity outside (0, 1). */
/* Recycling dead Gaussians, in place ([GS] "Densification: cloning the busy
 * blobs, recycling the dead", the variant with a fixed count). Among the first
 * n Gaussians, dead ones (opacity < dead_opacity) and donors (opacity >
 * donor_opacity) are found from the logits (decided in float64); the donors are
 * ranked largest first (largest log-scale, ties by index) and the j-th dead
 * Gaussian in index order is paired with the j-th donor, for j < min(dead,
 * donors, max_pairs). For each pair (d, b): slot d becomes a copy of b placed
 * at mean_b + R(q_b) diag(exp(log_scales_b)) z_j, with z_j = normals[3j..3j+2]
 * (DEVICE, float32 N(0, 1) draws supplied by the caller); both d and b take
 * log-scales log_scales_b - ln 1.6 ("both halves shrink"); both restart their
 * Adam moments (m and v zeroed in every group). Every other slot is left as
 * it was. params, m and v are the planar buffers of the parameters and of the
 * two Adam moments (mutable, same layout as gs_params, n_pad columns), updated
 * in place. The number of pairs made is written to the HOST int64 *n_pairs
 * (the call waits on the stream once to read the counts). It uses the
 * context's sort scratch, so the camera in flight is discarded (call
 * gs_preprocess again). Errors: GS_ERR_INVALID_ARG for NULL or misaligned
 * pointers, n > max_gaussians, n_pad < n or not a multiple of 4, sh_degree
 * outside 0..3, max_pairs < 0 (or > 0 with NULL normals), or thresholds not
 * satisfying 0 < dead_opacity < donor_opacity < 1; GS_ERR_CUDA if a launch or
 * the scratch allocation fails. */
gs_status gs_relocate(gs_ctx *ctx, const gs_grads *params, const gs_grads *m, const gs_grads *v, int64_t n,
                      int64_t n_pad, int32_t sh_degree, const float *normals, int64_t max_pairs,
                      float dead_opacity, float donor_opacity, int64_t *n_pairs, void *stream);

gs_status gs_opacity_reset(float *opacity_logits, float *m_logits, float *v_logits, int64_t n,
                           float max_opacity, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GS_API_H */
