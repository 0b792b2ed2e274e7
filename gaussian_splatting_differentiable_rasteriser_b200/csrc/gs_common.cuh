// Shared device constants, layouts and helpers of the sm_100a rasteriser.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gs {

constexpr int kTile = 16;               // 16x16-pixel screen tiles
constexpr int kTilePixels = kTile * kTile;
constexpr float kAlphaMax = 0.99f;      // alpha cap
constexpr float kAlphaMin = 1.0f / 255.0f;  // contributions below are skipped
constexpr float kTMin = 1e-4f;          // stop once T falls below this
constexpr double kDilation = 0.3;       // px^2 added to the screen covariance diagonal
constexpr float kDilationF = 0.3f;
constexpr double kRadiusSigmas = 3.0;   // sqrt(2 * 4.5): the falloff cut E_CUT = 4.5
constexpr float kLog2e = 1.4426950408889634f;

// Per-Gaussian screen state written by the preprocess and gathered by the
// blend kernels: 48 bytes, three 16-byte vectors, with the conic and opacity
// already in the form the exponent needs: alpha = min(0.99, 2^p),
//   p = A' dx^2 + B' dx dy + C' dy^2 + log2(o),
//   A' = -A log2(e) / 2, B' = -B log2(e), C' = -C log2(e) / 2
// for the conic (A, B, C) (e = A dx^2 / 2 + B dx dy + C dy^2 / 2).
//   a = (u, v, hx, hy)   hx, hy: conservative half-widths of the box holding
//                        every pixel where o exp(-e) >= 1/255 (negative if none)
//   b = (A', B', C', log2(o))
//   c = (r, g, b, o)
// The box test of the blend needs only a; b and c are gathered for the
// entries that pass it.
struct alignas(16) Screen {
  float4 a, b, c;
};

// Scale between the natural conic entries and the stored exponent form.
constexpr float kConicToExpAC = -0.5f * 1.4426950408889634f;  // A' = A * this (also C)
constexpr float kConicToExpB = -1.4426950408889634f;          // B' = B * this
__device__ __forceinline__ float conic_A(const Screen& s) { return s.b.x / kConicToExpAC; }
__device__ __forceinline__ float conic_B(const Screen& s) { return s.b.y / kConicToExpB; }
__device__ __forceinline__ float conic_C(const Screen& s) { return s.b.z / kConicToExpAC; }
__device__ __forceinline__ float screen_opacity(const Screen& s) { return s.c.w; }

// Raw per-Gaussian screen-gradient sums accumulated by the blend backward
// (12 floats, 9 used). With w = dL/dalpha * o exp(-e) summed over pixels:
//   [0] sum w        [1] sum w dx     [2] sum w dy
//   [3] sum w dx^2   [4] sum w dx dy  [5] sum w dy^2
//   [6..8] dL/d(r, g, b)
// The projection backward turns them into dL/d(mean2d, conic, opacity).
constexpr int kGradStride = 12;

// Deterministic mode keeps the 9 raw sums as 64-bit integers in 2^-40 fixed
// point, kFixedStride per Gaussian.
constexpr int kFixedStride = 9;
constexpr double kFixedScale = 1099511627776.0;      // 2^40
constexpr double kFixedClamp = 4611686018427387904.0;  // 2^62

// Camera in the form the kernels take it (by value).
struct CamArgs {
  int width, height, tiles_x, tiles_y;
  float fx, fy, cx, cy;
  float R[9];
  float t[3];
  float campos[3];
  float bg[3];
  float near_z;
};

// Device-side error word: kernels that give up on a bounded wait or detect an
// out-of-range index OR a code into it and skip the access.
enum DeviceError : uint32_t {
  kErrIndexRange = 2u,
  kErrCopyTimeout = 4u,
};

__device__ __forceinline__ void record_error(uint32_t* err, uint32_t code) {
  if (err) atomicOr(err, code);
}

// Pixel of thread `tid` inside a 16x16 tile: warp w covers an 8x4 block
// (two blocks across, four down), lane l its (l % 8, l / 8) pixel.
__device__ __forceinline__ void tile_pixel(int tid, int& x, int& y) {
  int w = tid >> 5, l = tid & 31;
  x = ((w & 1) << 3) + (l & 7);
  y = ((w >> 1) << 2) + (l >> 3);
}

}  // namespace gs
