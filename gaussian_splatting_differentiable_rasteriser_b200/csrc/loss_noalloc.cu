// A variant of the fused loss entry point that allocates nothing.
//
// Some callers cannot call cudaMalloc at the point where they need the loss:
// a host application whose own allocator owns the GPU's memory and gives the
// library device pointers for inputs and outputs but no allocator, and
// real-time loops whose memory is fixed after start-up (cudaMalloc can
// synchronise the device and stall such a loop). For
// them, gs_loss_l1_dssim_noalloc runs the same loss kernel as
// gs_loss_l1_dssim, with the kernel's scratch (one pair of float64 partial
// sums per CTA and the completion counter) in file-scope __device__ arrays of
// fixed size instead of in a context.
//
// The arrays are part of the library image: every GPU that loads the library
// holds them (about 0.2 MB) until the process exits. In host code the array
// names are host-side stand-ins, not device addresses, so the device address
// is taken once per device with cudaGetSymbolAddress while that device is
// current, and that address is what the kernel receives. The first call on a
// device does that lookup, so it should come before any stream capture. All
// calls on a device share the arrays: calls that overlap on the GPU race.
#include <cmath>
#include <mutex>

#include "gs_api.h"
#include "gs_kernels.cuh"

namespace gs {
int64_t loss_num_blocks(int height, int width);
}

namespace {

// Largest image the variant accepts: 4096 x 4096 (one loss CTA per channel
// and 32 x 128 strip, so 3 * 128 * 32 CTAs).
constexpr int kNoAllocMaxSide = 4096;
constexpr int64_t kNoAllocMaxBlocks = gs::loss_blocks(kNoAllocMaxSide, kNoAllocMaxSide);

static __device__ __align__(256) double g_loss_partials[2 * kNoAllocMaxBlocks];
static __device__ __align__(256) uint32_t g_loss_counter[1];

constexpr int kMaxDevices = 64;

struct DeviceScratch {
  double* partials = nullptr;
  uint32_t* counter = nullptr;
  bool ready = false;
};

DeviceScratch g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

// Device addresses of the scratch arrays on the current device (looked up on
// the first call on each device).
cudaError_t scratch_for_current_device(DeviceScratch& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  DeviceScratch& s = g_scratch[dev];
  if (!s.ready) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_loss_partials)) != cudaSuccess) return e;
    s.partials = static_cast<double*>(p);
    if ((e = cudaGetSymbolAddress(&p, g_loss_counter)) != cudaSuccess) return e;
    s.counter = static_cast<uint32_t*>(p);
    s.ready = true;
  }
  out = s;
  return cudaSuccess;
}

}  // namespace

extern "C" gs_status gs_loss_l1_dssim_noalloc(const float* image_chw, const float* target_chw,
                                              int32_t height, int32_t width, float lambda,
                                              double* loss_out, float* dloss_dimage, void* stream) {
  if (height <= 0 || width <= 0) return GS_ERR_INVALID_ARG;
  if (height > kNoAllocMaxSide || width > kNoAllocMaxSide ||
      gs::loss_num_blocks(height, width) > kNoAllocMaxBlocks)
    return GS_ERR_CAPACITY;
  auto aligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (!image_chw || !target_chw || !loss_out || !aligned(image_chw, 4) || !aligned(target_chw, 4) ||
      !aligned(loss_out, 8) || (dloss_dimage && !aligned(dloss_dimage, 4)))
    return GS_ERR_INVALID_ARG;
  if (!(lambda == lambda) || lambda > 3.4e38f || lambda < -3.4e38f) return GS_ERR_INVALID_ARG;
  DeviceScratch s;
  if (scratch_for_current_device(s) != cudaSuccess) return GS_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The counter must start at zero; a previous call leaves it at zero, but a
  // call interrupted by an error may not have, so clear it every time.
  if (cudaMemsetAsync(s.counter, 0, sizeof(uint32_t), st) != cudaSuccess) return GS_ERR_CUDA;
  gs::LossArgs a;
  a.x = image_chw;
  a.y = target_chw;
  a.height = height;
  a.width = width;
  a.lambda = lambda;
  double g[11], sum = 0.0;
  for (int i = 0; i < 11; ++i) sum += (g[i] = std::exp(-((i - 5) * (i - 5)) / (2.0 * 1.5 * 1.5)));
  for (int i = 0; i < 11; ++i) a.window[i] = static_cast<float>(g[i] / sum);
  a.dx = dloss_dimage;
  a.partials = s.partials;
  a.counter = s.counter;
  a.out = loss_out;
  return gs::launch_loss(a, st) == cudaSuccess ? GS_OK : GS_ERR_CUDA;
}
