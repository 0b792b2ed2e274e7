// Float64 CPU oracle of the differentiable tile-based Gaussian-splat rasteriser.
//
// TEST INFRASTRUCTURE ONLY. The tests, the package smoke check and the CPU
// baseline leg of the benchmark are the only code allowed to load this
// library. It shares no code, header, table or constant generator with the
// CUDA path, and nothing on the CUDA path calls it.
//
// What it computes, step by step, in the order and notation of the pages:
//   * preprocess  - "Gaussian splatting training" study notes (bailiping.com),
//                   slides on the parametrisation (log-scales, logit, normalised
//                   quaternion) and "J is the 2 x 3 Jacobian of perspective
//                   projection" (J, Sigma' = J W Sigma W^T J^T, +0.3 px^2);
//                   "How a computer rebuilds a real place ... Gaussian Splats"
//                   (taosengine.com), section "Flattening a 3D blob into a 2D
//                   oval (EWA projection)" (conic, radius, tile rect) and
//                   section "Spherical harmonics: color that changes with
//                   viewing angle" (view direction, SH colour, clamp at 0).
//   * tile lists  - same page, section "Why tiling, and the five stages":
//                   16x16 tiles, per-tile lists ordered near to far, equal keys
//                   broken by the smaller id. Here a library sort on the tuple
//                   (tile, float32 depth bits, id).
//   * blend       - same page, section "The painting itself: front-to-back
//                   alpha compositing"; study notes, slide on alpha (cap 0.99,
//                   skip below 1/255, stop when nearly opaque) and the
//                   background weight.
//   * loss        - study notes, slides on the loss (0.8 L1 + 0.2 (1 - SSIM)),
//                   L1 (mean over 3HW, zero subgradient at zero residual) and
//                   SSIM (11x11 Gaussian window, sigma 1.5, C1 = 0.01^2,
//                   C2 = 0.03^2, zero padding, mean over pixels and channels).
//   * backward    - study notes, slide "r is the RGB loss gradient":
//                   dI/dalpha_i = T_i (c_i - C_tail), dI/dc_i = T_i alpha_i,
//                   with the per-pixel list of contributors stored explicitly
//                   (the plain approach the "Differentiable rasterisation"
//                   page, section "Why the naive backward pass doesn't scale",
//                   describes). Every other partial derivative (alpha w.r.t.
//                   the screen parameters, the whole projection w.r.t. the
//                   stored parameters including the view-direction path, SSIM
//                   w.r.t. its window moments) is taken exactly by forward-mode
//                   dual numbers through the forward code above.
//   * Adam        - taosengine page, Adam paragraph after "Proving the blame is
//                   right": moments, bias correction, p -= lr mh/(sqrt(vh)+eps).
//
// Readings where the pages are silent: pixel (i, j) sits at (i, j); camera axes
// x right, y down, z forward with p_c = R p + t; cull when Z <= near_z;
// r = 3 sqrt(lambda_max) (the E_CUT = 4.5 cap); the Gaussian that drops T
// below 1e-4 is blended and then the walk stops; the DC coefficient is the base
// RGB (basis 1); the view direction is normalize(p - campos); depth keys are
// float32(Z) with Z evaluated as ((R20 x + R21 y) + R22 z) + t2 in float64.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -shared -fPIC (see build.py).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

constexpr double kPi = 3.14159265358979323846;
constexpr int kTile = 16;
constexpr double kDilation = 0.3;
constexpr double kAlphaMax = 0.99;
constexpr double kAlphaMin = 1.0 / 255.0;
constexpr double kTMin = 1e-4;
constexpr double kRadiusSigmas = 3.0;  // sqrt(2 * E_CUT), E_CUT = 4.5

// ------------------------------------------------------------------ duals --
// Forward-mode dual numbers: value plus N partial derivatives.
template <int N>
struct Dual {
  double v;
  double d[N];
  Dual() : v(0.0) {
    for (int i = 0; i < N; ++i) d[i] = 0.0;
  }
  Dual(double x) : v(x) {  // NOLINT: implicit constants are intended
    for (int i = 0; i < N; ++i) d[i] = 0.0;
  }
};

template <int N>
Dual<N> seed(double x, int i) {
  Dual<N> r(x);
  r.d[i] = 1.0;
  return r;
}

inline double val(double x) { return x; }
template <int N>
double val(const Dual<N>& x) { return x.v; }

template <int N>
Dual<N> operator+(const Dual<N>& a, const Dual<N>& b) {
  Dual<N> r(a.v + b.v);
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] + b.d[i];
  return r;
}
template <int N>
Dual<N> operator-(const Dual<N>& a, const Dual<N>& b) {
  Dual<N> r(a.v - b.v);
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] - b.d[i];
  return r;
}
template <int N>
Dual<N> operator-(const Dual<N>& a) {
  Dual<N> r(-a.v);
  for (int i = 0; i < N; ++i) r.d[i] = -a.d[i];
  return r;
}
template <int N>
Dual<N> operator*(const Dual<N>& a, const Dual<N>& b) {
  Dual<N> r(a.v * b.v);
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] * b.v + a.v * b.d[i];
  return r;
}
template <int N>
Dual<N> operator/(const Dual<N>& a, const Dual<N>& b) {
  Dual<N> r(a.v / b.v);
  for (int i = 0; i < N; ++i) r.d[i] = (a.d[i] * b.v - a.v * b.d[i]) / (b.v * b.v);
  return r;
}
template <int N>
Dual<N> operator+(const Dual<N>& a, double b) { return a + Dual<N>(b); }
template <int N>
Dual<N> operator+(double a, const Dual<N>& b) { return Dual<N>(a) + b; }
template <int N>
Dual<N> operator-(const Dual<N>& a, double b) { return a - Dual<N>(b); }
template <int N>
Dual<N> operator-(double a, const Dual<N>& b) { return Dual<N>(a) - b; }
template <int N>
Dual<N> operator*(const Dual<N>& a, double b) { return a * Dual<N>(b); }
template <int N>
Dual<N> operator*(double a, const Dual<N>& b) { return Dual<N>(a) * b; }
template <int N>
Dual<N> operator/(const Dual<N>& a, double b) { return a / Dual<N>(b); }
template <int N>
Dual<N> operator/(double a, const Dual<N>& b) { return Dual<N>(a) / b; }

template <int N>
Dual<N> exp(const Dual<N>& a) {
  double e = std::exp(a.v);
  Dual<N> r(e);
  for (int i = 0; i < N; ++i) r.d[i] = e * a.d[i];
  return r;
}
template <int N>
Dual<N> sqrt(const Dual<N>& a) {
  double s = std::sqrt(a.v);
  Dual<N> r(s);
  for (int i = 0; i < N; ++i) r.d[i] = a.d[i] / (2.0 * s);
  return r;
}
using std::exp;
using std::sqrt;

// ------------------------------------------------------ spherical harmonics --
// Real spherical harmonics up to degree 3, derived here from their closed
// form rather than taken from a table:
//   P_l(z) by Rodrigues' formula, Q_l^m(z) = (-1)^m d^m P_l / dz^m
//   (the Condon-Shortley phase), K_l^m = sqrt((2l+1)/(4 pi) (l-m)!/(l+m)!),
//   Y_{l,m} = sqrt2 K Q(z) Re((x+iy)^m)   for m > 0,
//           = sqrt2 K Q(z) Im((x+iy)^|m|) for m < 0,
//           = K Q(z)                      for m = 0,
// stored at k = l^2 + l + m. With this phase the degree-1 functions come out
// as (-y, z, -x) times 0.4886025, the pattern the taosengine page prints.
// k = 0 is the base colour with basis 1 (the pages never print the DC
// constant; the stored DC coefficient is the RGB itself).
struct ShBasis {
  double q[4][4][7];  // [l][m][power of z]
  double k[4][4];     // normalisation, including sqrt2 for m > 0

  ShBasis() {
    std::memset(q, 0, sizeof(q));
    for (int l = 0; l <= 3; ++l) {
      // (z^2 - 1)^l as ascending coefficients.
      double poly[7] = {0, 0, 0, 0, 0, 0, 0};
      for (int j = 0; j <= l; ++j) poly[2 * j] = binom(l, j) * ((l - j) % 2 ? -1.0 : 1.0);
      // l-th derivative, scaled by 1 / (2^l l!).
      for (int r = 0; r < l; ++r) differentiate(poly);
      double scale = 1.0 / (std::pow(2.0, l) * fact(l));
      for (double& c : poly) c *= scale;
      // Q_l^m: m further derivatives with the (-1)^m phase.
      double pm[7];
      std::memcpy(pm, poly, sizeof(pm));
      for (int m = 0; m <= l; ++m) {
        for (int p = 0; p < 7; ++p) q[l][m][p] = (m % 2 ? -1.0 : 1.0) * pm[p];
        k[l][m] = std::sqrt((2.0 * l + 1.0) / (4.0 * kPi) * fact(l - m) / fact(l + m)) *
                  (m > 0 ? std::sqrt(2.0) : 1.0);
        differentiate(pm);
      }
    }
  }
  static double fact(int n) {
    double r = 1.0;
    for (int i = 2; i <= n; ++i) r *= i;
    return r;
  }
  static double binom(int n, int k) { return fact(n) / (fact(k) * fact(n - k)); }
  static void differentiate(double* p) {
    for (int i = 0; i < 6; ++i) p[i] = p[i + 1] * (i + 1);
    p[6] = 0.0;
  }

  // out[k] for k < (degree+1)^2 at unit direction (x, y, z).
  template <class S>
  void eval(int degree, const S& x, const S& y, const S& z, S* out) const {
    out[0] = S(1.0);
    for (int l = 1; l <= degree; ++l) {
      for (int m = -l; m <= l; ++m) {
        int am = m < 0 ? -m : m;
        S qz(0.0);
        for (int p = 6; p >= 0; --p) qz = qz * z + q[l][am][p];
        S re(1.0), im(0.0);
        for (int i = 0; i < am; ++i) {
          S nre = re * x - im * y;
          S nim = re * y + im * x;
          re = nre;
          im = nim;
        }
        S v = (m == 0) ? qz : (m > 0 ? qz * re : qz * im);
        out[l * l + l + m] = k[l][am] * v;
      }
    }
  }
};

const ShBasis& sh_basis() {
  static const ShBasis b;
  return b;
}

}  // namespace

extern "C" {

// Camera given to the oracle. All values are the float32 numbers the CUDA
// path receives, widened to float64.
struct or_camera {
  int32_t width, height;
  double fx, fy, cx, cy;
  double R[9];  // world -> camera rotation, row-major
  double t[3];
  double campos[3];
  double bg[3];
  double near_z;
};

}  // extern "C"

namespace {

// Screen-space result of one Gaussian, as a function of its parameters.
template <class S>
struct Proj {
  S u, v;     // projected mean (pixels)
  S a, b, c;  // dilated screen covariance Sigma' = [[a, b], [b, c]]
  S A, B, C;  // conic = Sigma'^-1 = [[A, B], [B, C]]
  S o;        // opacity
  S rgb[3];   // clamped colour
};

// Non-differentiable by-products of the projection.
struct Aux {
  double Z = 0.0;
  float depth_key = 0.0f;
  double lmax = 0.0, radius = 0.0;
  int32_t rect[4] = {0, 0, -1, -1};  // x0, y0, x1, y1 inclusive tile indices
  int32_t touched = 0;
  bool clamped[3] = {false, false, false};
  double dir[3] = {0.0, 0.0, 0.0};
  double Y[16] = {0};
};

template <class Cam>
int tiles_x(const Cam& cam) { return (cam.width + kTile - 1) / kTile; }
template <class Cam>
int tiles_y(const Cam& cam) { return (cam.height + kTile - 1) / kTile; }

// A camera whose pose is a function of a perturbation (dual numbers): the
// projection below is written once for both camera types.
template <class S>
struct PoseCamera {
  int32_t width, height;
  double fx, fy, cx, cy;
  S R[9];
  S t[3];
  S campos[3];
  double near_z;
};

// Rotation matrix of the normalised quaternion (w, x, y, z), row-major.
template <class S>
void quat_to_rot(const S q[4], S R[9]) {
  S w = q[0], x = q[1], y = q[2], z = q[3];
  R[0] = 1.0 - 2.0 * (y * y + z * z);
  R[1] = 2.0 * (x * y - w * z);
  R[2] = 2.0 * (x * z + w * y);
  R[3] = 2.0 * (x * y + w * z);
  R[4] = 1.0 - 2.0 * (x * x + z * z);
  R[5] = 2.0 * (y * z - w * x);
  R[6] = 2.0 * (x * z - w * y);
  R[7] = 2.0 * (y * z + w * x);
  R[8] = 1.0 - 2.0 * (x * x + y * y);
}

// Sigma = M M^T with M = R(q / |q|) diag(exp(ls)).
template <class S>
void covariance3d(const S ls[3], const S q[4], S Sigma[9]) {
  S qn = sqrt(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
  S qh[4] = {q[0] / qn, q[1] / qn, q[2] / qn, q[3] / qn};
  S R[9];
  quat_to_rot(qh, R);
  S s[3] = {exp(ls[0]), exp(ls[1]), exp(ls[2])};
  S M[9];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) M[3 * i + j] = R[3 * i + j] * s[j];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) {
      S acc(0.0);
      for (int k = 0; k < 3; ++k) acc = acc + M[3 * i + k] * M[3 * j + k];
      Sigma[3 * i + j] = acc;
    }
}

// One Gaussian through the preprocess. Returns false if it is culled (behind
// the near plane, degenerate screen covariance, or a tile rect that misses the
// image), in which case it touches no tile.
//
// With opacity_rect the tile rect uses the opacity-aware radius of "How a
// computer rebuilds a real place ... Gaussian Splats", section "Why tiling,
// and the five stages" (the code after the five stages): the falloff cut is
// E = min(4.5, ln(max(o / alpha_min, 1.0001))) with alpha_min = 1/255 and no
// compensation factor, and r = sqrt(2 E) sqrt(lambda_max). Beyond r along
// the long axis o exp(-e) < 1/255, so the tiles it drops hold no contribution.
//
// With mip_comp the opacity is multiplied by the compensation factor that
// section "Flattening a 3D blob into a 2D oval (EWA projection)" attributes
// to Mip-Splatting (its alpha is min(0.99, opacity * comp * exp(-e)), and the
// opacity-aware radius uses opacity * comp). The pages print no formula; the
// factor is the 2D Mip filter of Mip-Splatting (Yu et al., "Mip-Splatting:
// Alias-free 3D Gaussian Splatting", CVPR 2024), comp = sqrt(det V /
// det(V + s I)), with V the screen covariance before dilation and s the
// pages' 0.3 px^2 dilation: the dilated splat then carries the integrated
// weight of the undilated one, so a splat much smaller than a pixel does not
// gain weight from the dilation. comp = 0 when det V <= 0.
template <class S, class Cam>
bool project(const Cam& cam, const S p[3], const S ls[3], const S q[4], const S& logit,
             const double* sh, int64_t sh_stride, int active_degree, Proj<S>& P, Aux& X,
             bool opacity_rect = false, bool mip_comp = false) {
  X = Aux();
  const auto* R = cam.R;
  // p_c = R p + t, each row summed left to right.
  S pc[3];
  for (int i = 0; i < 3; ++i)
    pc[i] = ((R[3 * i + 0] * p[0] + R[3 * i + 1] * p[1]) + R[3 * i + 2] * p[2]) + cam.t[i];
  X.Z = val(pc[2]);
  X.depth_key = static_cast<float>(X.Z);
  if (!(X.Z > cam.near_z)) return false;

  S Sigma[9];
  covariance3d(ls, q, Sigma);

  // J at p_c, then T = J W with W the camera rotation.
  S X_ = pc[0], Y_ = pc[1], Z_ = pc[2];
  S J[6] = {cam.fx / Z_, S(0.0), -cam.fx * X_ / (Z_ * Z_),
            S(0.0), cam.fy / Z_, -cam.fy * Y_ / (Z_ * Z_)};
  S T[6];
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 3; ++j) {
      S acc(0.0);
      for (int k = 0; k < 3; ++k) acc = acc + J[3 * i + k] * R[3 * k + j];
      T[3 * i + j] = acc;
    }
  // Sigma' = T Sigma T^T + 0.3 I
  S V[4];
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 2; ++j) {
      S acc(0.0);
      for (int k = 0; k < 3; ++k)
        for (int l = 0; l < 3; ++l) acc = acc + T[3 * i + k] * Sigma[3 * k + l] * T[3 * j + l];
      V[2 * i + j] = acc;
    }
  P.a = V[0] + kDilation;
  P.b = V[1];
  P.c = V[3] + kDilation;
  S det = P.a * P.c - P.b * P.b;
  if (!(val(det) > 0.0)) return false;
  P.A = P.c / det;
  P.B = -P.b / det;
  P.C = P.a / det;
  S comp(1.0);
  if (mip_comp) {
    S det0 = V[0] * V[3] - V[1] * V[1];
    comp = val(det0) > 0.0 ? sqrt(det0 / det) : S(0.0);
  }

  P.u = cam.fx * X_ / Z_ + cam.cx;
  P.v = cam.fy * Y_ / Z_ + cam.cy;

  // Radius from the largest eigenvalue of the dilated covariance.
  double mid = 0.5 * (val(P.a) + val(P.c));
  double dt = val(det);
  X.lmax = mid + std::sqrt(std::max(mid * mid - dt, 0.0));
  X.radius = kRadiusSigmas * std::sqrt(X.lmax);
  if (opacity_rect) {
    const double o = 1.0 / (1.0 + std::exp(-val(logit))) * val(comp);
    const double e_cut = std::min(4.5, std::log(std::max(o * 255.0, 1.0001)));
    X.radius = std::sqrt(2.0 * e_cut) * std::sqrt(X.lmax);
  }
  // Tiles whose pixel square [16 tx, 16 tx + 15] meets [u - r, u + r].
  double u = val(P.u), v = val(P.v), r = X.radius;
  int tx0 = static_cast<int>(std::ceil((u - r - (kTile - 1)) / kTile));
  int tx1 = static_cast<int>(std::floor((u + r) / kTile));
  int ty0 = static_cast<int>(std::ceil((v - r - (kTile - 1)) / kTile));
  int ty1 = static_cast<int>(std::floor((v + r) / kTile));
  tx0 = std::max(tx0, 0);
  ty0 = std::max(ty0, 0);
  tx1 = std::min(tx1, tiles_x(cam) - 1);
  ty1 = std::min(ty1, tiles_y(cam) - 1);
  X.rect[0] = tx0;
  X.rect[1] = ty0;
  X.rect[2] = tx1;
  X.rect[3] = ty1;
  if (tx0 > tx1 || ty0 > ty1) return false;
  X.touched = (tx1 - tx0 + 1) * (ty1 - ty0 + 1);

  P.o = 1.0 / (1.0 + exp(-logit)) * comp;

  // View-dependent colour at the direction from the camera to the Gaussian.
  S d[3] = {p[0] - cam.campos[0], p[1] - cam.campos[1], p[2] - cam.campos[2]};
  S dn = sqrt(d[0] * d[0] + d[1] * d[1] + d[2] * d[2]);
  S dir[3] = {d[0] / dn, d[1] / dn, d[2] / dn};
  for (int i = 0; i < 3; ++i) X.dir[i] = val(dir[i]);
  S Y[16];
  sh_basis().eval(active_degree, dir[0], dir[1], dir[2], Y);
  int nk = (active_degree + 1) * (active_degree + 1);
  for (int k = 0; k < nk; ++k) X.Y[k] = val(Y[k]);
  for (int ch = 0; ch < 3; ++ch) {
    S col(0.0);
    for (int k = 0; k < nk; ++k) col = col + sh[(ch * 16 + k) * sh_stride] * Y[k];
    if (val(col) < 0.0) {
      P.rgb[ch] = S(0.0);
      X.clamped[ch] = true;
    } else {
      P.rgb[ch] = col;
    }
  }
  return true;
}

struct Entry {
  int32_t tile;
  uint32_t depth_bits;
  int32_t id;
  bool operator<(const Entry& o) const {
    if (tile != o.tile) return tile < o.tile;
    if (depth_bits != o.depth_bits) return depth_bits < o.depth_bits;
    return id < o.id;
  }
};

// Per-Gaussian screen state in float64: u, v, A, B, C, o, r, g, b.
constexpr int kScreen = 9;

struct Contribution {
  int32_t id;
  int32_t pos;      // position inside the tile list
  double alpha;     // after the 0.99 cap
  double T;         // transmittance in front of this Gaussian
  Dual<6> alpha_d;  // alpha as a function of (u, v, A, B, C, o); zero when capped
};

struct PixelResult {
  double rgb[3];
  double T;
  int32_t n_contrib;  // 1 + list position of the last contributor, 0 if none
  bool ambiguous;     // some decision fell within a hair of its threshold
  int64_t evaluated;  // list entries evaluated
  int64_t contributions;  // entries that passed the alpha floor
};

struct Ctx {
  or_camera cam{};
  int64_t n = 0, n_pad = 0;
  int sh_degree = 0, active_degree = 0;
  std::vector<double> means, ls, quats, logits, sh;  // planar float64 copies
  std::vector<double> screen;                        // n x 9
  std::vector<double> cov2d;                         // n x 3 (a, b, c)
  std::vector<Aux> aux;
  std::vector<Entry> entries;            // sorted
  std::vector<int64_t> range_lo, range_hi;  // per tile, [lo, hi)
  bool opacity_rect = false;             // opacity-aware tile rect (see project)
  bool mip_comp = false;                 // Mip-Splatting compensation factor (see project)
};

// Margins used to flag float32/float64 threshold ambiguity.
constexpr double kAlphaMargin = 1e-6;
constexpr double kTMargin = 1e-3;  // relative

// With flip != 0 the walk is replayed with some of its near-threshold
// decisions taken the other way: the k-th such decision met (an alpha within
// kAlphaMargin of 1/255, or a transmittance within kTMargin of 1e-4, counted
// in walk order) is flipped when bit k of `flip` is set. A float32 renderer
// may take any of those decisions either way; the replays are the results it
// can then give. *n_amb receives the number of such decisions met.
void walk_pixel(const Ctx& c, int px, int py, PixelResult& out, std::vector<Contribution>* list,
                uint32_t flip = 0, int* n_amb = nullptr) {
  const or_camera& cam = c.cam;
  int tile = (py / kTile) * tiles_x(cam) + (px / kTile);
  double T = 1.0;
  double rgb[3] = {0.0, 0.0, 0.0};
  out.n_contrib = 0;
  out.ambiguous = false;
  out.evaluated = 0;
  out.contributions = 0;
  int amb = 0;
  if (list) list->clear();
  for (int64_t i = c.range_lo[tile]; i < c.range_hi[tile]; ++i) {
    int32_t g = c.entries[i].id;
    const double* s = &c.screen[static_cast<size_t>(g) * kScreen];
    ++out.evaluated;
    double dx = static_cast<double>(px) - s[0];
    double dy = static_cast<double>(py) - s[1];
    double e = 0.5 * (s[2] * dx * dx + s[4] * dy * dy) + s[3] * dx * dy;
    double a = s[5] * std::exp(-e);
    double alpha = a > kAlphaMax ? kAlphaMax : a;
    bool skip = alpha < kAlphaMin;
    if (std::fabs(alpha - kAlphaMin) < kAlphaMargin) {
      out.ambiguous = true;
      if (amb < 32 && ((flip >> amb) & 1u)) skip = !skip;
      ++amb;
    }
    if (skip) continue;
    ++out.contributions;
    if (list) {
      // The same alpha as a function of (u, v, A, B, C, o), for the backward.
      Dual<6> u = seed<6>(s[0], 0), v = seed<6>(s[1], 1);
      Dual<6> A = seed<6>(s[2], 2), B = seed<6>(s[3], 3), C = seed<6>(s[4], 4);
      Dual<6> o = seed<6>(s[5], 5);
      Dual<6> ddx = static_cast<double>(px) - u;
      Dual<6> ddy = static_cast<double>(py) - v;
      Dual<6> de = 0.5 * (A * ddx * ddx + C * ddy * ddy) + B * ddx * ddy;
      Dual<6> da = o * exp(-de);
      Dual<6> dalpha = a > kAlphaMax ? Dual<6>(kAlphaMax) : da;
      list->push_back({g, static_cast<int32_t>(i - c.range_lo[tile]), alpha, T, dalpha});
    }
    for (int ch = 0; ch < 3; ++ch) rgb[ch] += T * alpha * s[6 + ch];
    double Tn = T * (1.0 - alpha);
    out.n_contrib = static_cast<int32_t>(i - c.range_lo[tile]) + 1;
    bool stop = Tn < kTMin;
    if (std::fabs(Tn - kTMin) < kTMargin * kTMin) {
      out.ambiguous = true;
      if (amb < 32 && ((flip >> amb) & 1u)) stop = !stop;
      ++amb;
    }
    T = Tn;
    if (stop) break;
  }
  for (int ch = 0; ch < 3; ++ch) out.rgb[ch] = rgb[ch] + T * cam.bg[ch];
  out.T = T;
  if (n_amb) *n_amb = amb;
}

template <class In>
void load_params(Ctx& c, int64_t n, int64_t n_pad, int sh_degree, const In* means, const In* ls,
                 const In* quats, const In* logits, const In* sh) {
  c.n = n;
  c.n_pad = n_pad;
  c.sh_degree = sh_degree;
  int K = (sh_degree + 1) * (sh_degree + 1);
  c.means.assign(means, means + 3 * n_pad);
  c.ls.assign(ls, ls + 3 * n_pad);
  c.quats.assign(quats, quats + 4 * n_pad);
  c.logits.assign(logits, logits + n_pad);
  // SH widened to a [3][16][n_pad] table so degree-3 indexing is uniform.
  c.sh.assign(static_cast<size_t>(3) * 16 * n_pad, 0.0);
  for (int ch = 0; ch < 3; ++ch)
    for (int k = 0; k < K; ++k)
      for (int64_t i = 0; i < n_pad; ++i)
        c.sh[(static_cast<size_t>(ch) * 16 + k) * n_pad + i] =
            sh[(static_cast<size_t>(ch) * K + k) * n_pad + i];
}

void run_preprocess_and_sort(Ctx& c) {
  const int64_t n = c.n, np = c.n_pad;
  c.screen.assign(static_cast<size_t>(n) * kScreen, 0.0);
  c.cov2d.assign(static_cast<size_t>(n) * 3, 0.0);
  c.aux.assign(static_cast<size_t>(n), Aux());
  c.entries.clear();
  for (int64_t i = 0; i < n; ++i) {
    double p[3] = {c.means[i], c.means[np + i], c.means[2 * np + i]};
    double ls[3] = {c.ls[i], c.ls[np + i], c.ls[2 * np + i]};
    double q[4] = {c.quats[i], c.quats[np + i], c.quats[2 * np + i], c.quats[3 * np + i]};
    Proj<double> P;
    Aux& X = c.aux[i];
    bool ok = project<double>(c.cam, p, ls, q, c.logits[i], &c.sh[i], np, c.active_degree, P, X,
                              c.opacity_rect, c.mip_comp);
    if (!ok) {
      X.touched = 0;
      continue;
    }
    double* s = &c.screen[static_cast<size_t>(i) * kScreen];
    s[0] = P.u; s[1] = P.v; s[2] = P.A; s[3] = P.B; s[4] = P.C; s[5] = P.o;
    s[6] = P.rgb[0]; s[7] = P.rgb[1]; s[8] = P.rgb[2];
    c.cov2d[3 * i + 0] = P.a;
    c.cov2d[3 * i + 1] = P.b;
    c.cov2d[3 * i + 2] = P.c;
    uint32_t bits;
    std::memcpy(&bits, &X.depth_key, 4);
    for (int ty = X.rect[1]; ty <= X.rect[3]; ++ty)
      for (int tx = X.rect[0]; tx <= X.rect[2]; ++tx)
        c.entries.push_back({ty * tiles_x(c.cam) + tx, bits, static_cast<int32_t>(i)});
  }
  std::sort(c.entries.begin(), c.entries.end());
  int nt = tiles_x(c.cam) * tiles_y(c.cam);
  c.range_lo.assign(nt, 0);
  c.range_hi.assign(nt, 0);
  for (size_t i = 0; i < c.entries.size(); ++i) {
    int t = c.entries[i].tile;
    if (i == 0 || c.entries[i - 1].tile != t) c.range_lo[t] = static_cast<int64_t>(i);
    c.range_hi[t] = static_cast<int64_t>(i) + 1;
  }
}

// Backward through the blend for one pixel, given dL/dI at that pixel.
// Accumulates dL/d(u, v, A, B, C, o, r, g, b) per Gaussian.
void backward_pixel(const Ctx& c, const std::vector<Contribution>& list, const double g[3],
                    double* sgrad) {
  double tail[3] = {c.cam.bg[0], c.cam.bg[1], c.cam.bg[2]};
  for (int64_t i = static_cast<int64_t>(list.size()) - 1; i >= 0; --i) {
    const Contribution& k = list[i];
    const double* s = &c.screen[static_cast<size_t>(k.id) * kScreen];
    double* gs = &sgrad[static_cast<size_t>(k.id) * kScreen];
    double dalpha = 0.0;
    for (int ch = 0; ch < 3; ++ch) {
      dalpha += g[ch] * k.T * (s[6 + ch] - tail[ch]);  // dI/dalpha_i = T_i (c_i - C_tail)
      gs[6 + ch] += g[ch] * k.T * k.alpha;             // dI/dc_i = T_i alpha_i
    }
    for (int j = 0; j < 6; ++j) gs[j] += dalpha * k.alpha_d.d[j];
    for (int ch = 0; ch < 3; ++ch) tail[ch] = k.alpha * s[6 + ch] + (1.0 - k.alpha) * tail[ch];
  }
}

}  // namespace

extern "C" {

void* or_create() { return new Ctx(); }
void or_destroy(void* h) { delete static_cast<Ctx*>(h); }

// Options, set before or_set_scene: 1 = opacity-aware tile rect, 2 = the
// Mip-Splatting compensation factor in the opacity (values 0/1).
// Returns 0, or 1 for an unknown option.
int or_set_option(void* h, int32_t option, int32_t value) {
  Ctx& c = *static_cast<Ctx*>(h);
  if (option == 1) {
    c.opacity_rect = value != 0;
    return 0;
  }
  if (option == 2) {
    c.mip_comp = value != 0;
    return 0;
  }
  return 1;
}

// Loads the parameters (planar float32, see the scene layout) and the camera,
// then runs the preprocess and builds the sorted tile lists.
}  // extern "C"

namespace {

template <class In>
int set_scene(void* h, int64_t n, int64_t n_pad, int32_t sh_degree, int32_t active_degree,
              const In* means, const In* log_scales, const In* quats, const In* opacity_logits,
              const In* sh, const or_camera* cam) {
  Ctx& c = *static_cast<Ctx*>(h);
  if (n < 0 || n_pad < n || sh_degree < 0 || sh_degree > 3 || active_degree < 0 ||
      active_degree > sh_degree || cam->width <= 0 || cam->height <= 0)
    return 1;
  c.cam = *cam;
  c.active_degree = active_degree;
  load_params(c, n, n_pad, sh_degree, means, log_scales, quats, opacity_logits, sh);
  run_preprocess_and_sort(c);
  return 0;
}

}  // namespace

extern "C" {

int or_set_scene(void* h, int64_t n, int64_t n_pad, int32_t sh_degree, int32_t active_degree,
                 const float* means, const float* log_scales, const float* quats,
                 const float* opacity_logits, const float* sh, const or_camera* cam) {
  return set_scene<float>(h, n, n_pad, sh_degree, active_degree, means, log_scales, quats,
                          opacity_logits, sh, cam);
}

// The same with float64 parameters (used by the central-difference checks).
int or_set_scene_f64(void* h, int64_t n, int64_t n_pad, int32_t sh_degree,
                     int32_t active_degree, const double* means, const double* log_scales,
                     const double* quats, const double* opacity_logits, const double* sh,
                     const or_camera* cam) {
  return set_scene<double>(h, n, n_pad, sh_degree, active_degree, means, log_scales, quats,
                           opacity_logits, sh, cam);
}

// Screen state n x 9 (u, v, A, B, C, o, r, g, b), dilated covariance n x 3,
// depth n, float32 depth key n, radius n, rect n x 4, tiles touched n,
// clamp flags n x 3. Culled Gaussians report zeros and touched = 0.
void or_get_preprocess(void* h, double* screen, double* cov2d, double* depth, float* depth_key,
                       double* radius, int32_t* rect, int32_t* touched, uint8_t* clamped) {
  const Ctx& c = *static_cast<Ctx*>(h);
  for (int64_t i = 0; i < c.n; ++i) {
    const Aux& X = c.aux[i];
    if (screen)
      for (int j = 0; j < kScreen; ++j) screen[kScreen * i + j] = c.screen[kScreen * i + j];
    if (cov2d)
      for (int j = 0; j < 3; ++j) cov2d[3 * i + j] = c.cov2d[3 * i + j];
    if (depth) depth[i] = X.Z;
    if (depth_key) depth_key[i] = X.depth_key;
    if (radius) radius[i] = X.radius;
    if (rect)
      for (int j = 0; j < 4; ++j) rect[4 * i + j] = X.rect[j];
    if (touched) touched[i] = X.touched;
    if (clamped)
      for (int j = 0; j < 3; ++j) clamped[3 * i + j] = X.clamped[j] ? 1 : 0;
  }
}

int64_t or_num_entries(void* h) { return static_cast<int64_t>(static_cast<Ctx*>(h)->entries.size()); }

// Sorted entries (Gaussian id and tile per entry) and per-tile [lo, hi) ranges.
void or_get_sorted(void* h, int32_t* ids, int32_t* tiles, int64_t* ranges) {
  const Ctx& c = *static_cast<Ctx*>(h);
  for (size_t i = 0; i < c.entries.size(); ++i) {
    if (ids) ids[i] = c.entries[i].id;
    if (tiles) tiles[i] = c.entries[i].tile;
  }
  if (ranges)
    for (size_t t = 0; t < c.range_lo.size(); ++t) {
      ranges[2 * t] = c.range_lo[t];
      ranges[2 * t + 1] = c.range_hi[t];
    }
}

// Forward over the pixel rows [y0, y1) (full-size outputs, other rows untouched):
// image [3][H][W], final T [H][W], n_contrib [H][W], ambiguity flags [H][W];
// stats[0] = entries evaluated, stats[1] = contributions.
void or_render_rows(void* h, int32_t y0, int32_t y1, double* image, double* final_T,
                    int32_t* n_contrib, uint8_t* ambiguous, int64_t* stats) {
  const Ctx& c = *static_cast<Ctx*>(h);
  const int W = c.cam.width, H = c.cam.height;
  int64_t evaluated = 0, contributions = 0;
  y0 = std::max(y0, 0);
  y1 = std::min(y1, H);
  for (int py = y0; py < y1; ++py)
    for (int px = 0; px < W; ++px) {
      PixelResult r;
      walk_pixel(c, px, py, r, nullptr);
      size_t p = static_cast<size_t>(py) * W + px;
      for (int ch = 0; ch < 3; ++ch) image[static_cast<size_t>(ch) * H * W + p] = r.rgb[ch];
      if (final_T) final_T[p] = r.T;
      if (n_contrib) n_contrib[p] = r.n_contrib;
      if (ambiguous) ambiguous[p] = r.ambiguous ? 1 : 0;
      evaluated += r.evaluated;
      contributions += r.contributions;
    }
  if (stats) {
    stats[0] = evaluated;
    stats[1] = contributions;
  }
}

// Full-image forward (all rows).
void or_render(void* h, double* image, double* final_T, int32_t* n_contrib, uint8_t* ambiguous,
               int64_t* stats) {
  or_render_rows(h, 0, static_cast<Ctx*>(h)->cam.height, image, final_T, n_contrib, ambiguous, stats);
}

// Forward at a list of pixels only (for sampled checks at full size).
void or_render_pixels(void* h, int64_t npix, const int32_t* px, const int32_t* py, double* rgb,
                      double* T, int32_t* n_contrib, uint8_t* ambiguous) {
  const Ctx& c = *static_cast<Ctx*>(h);
  for (int64_t i = 0; i < npix; ++i) {
    PixelResult r;
    walk_pixel(c, px[i], py[i], r, nullptr);
    for (int ch = 0; ch < 3; ++ch) rgb[3 * i + ch] = r.rgb[ch];
    if (T) T[i] = r.T;
    if (n_contrib) n_contrib[i] = r.n_contrib;
    if (ambiguous) ambiguous[i] = r.ambiguous ? 1 : 0;
  }
}

// Replays of the forward at a list of pixels (test support for threshold
// decisions a float32 renderer may take either way): pixel i is walked with
// the near-threshold decisions in bit mask flip[i] flipped (see walk_pixel);
// n_amb[i] = the number of near-threshold decisions that walk met.
void or_render_pixels_replay(void* h, int64_t npix, const int32_t* px, const int32_t* py,
                             const uint32_t* flip, double* rgb, double* T, int32_t* n_contrib,
                             int32_t* n_amb) {
  const Ctx& c = *static_cast<Ctx*>(h);
  for (int64_t i = 0; i < npix; ++i) {
    PixelResult r;
    int amb = 0;
    walk_pixel(c, px[i], py[i], r, nullptr, flip[i], &amb);
    for (int ch = 0; ch < 3; ++ch) rgb[3 * i + ch] = r.rgb[ch];
    T[i] = r.T;
    n_contrib[i] = r.n_contrib;
    n_amb[i] = amb;
  }
}

// Blend backward over the pixel rows [y0, y1): ADDS each pixel's contribution to
// the screen gradient n x 9 (dL/du, dv, dA, dB, dC, d opacity, dr, dg, db);
// dL/dimage is [3][H][W], full size.
void or_blend_backward_rows(void* h, int32_t y0, int32_t y1, const double* dimage,
                            double* screen_grad) {
  const Ctx& c = *static_cast<Ctx*>(h);
  const int W = c.cam.width, H = c.cam.height;
  std::vector<Contribution> list;
  y0 = std::max(y0, 0);
  y1 = std::min(y1, H);
  for (int py = y0; py < y1; ++py)
    for (int px = 0; px < W; ++px) {
      PixelResult r;
      walk_pixel(c, px, py, r, &list);
      size_t p = static_cast<size_t>(py) * W + px;
      double g[3] = {dimage[p], dimage[static_cast<size_t>(H) * W + p],
                     dimage[2 * static_cast<size_t>(H) * W + p]};
      backward_pixel(c, list, g, screen_grad);
    }
}

// Projection backward of the Gaussians [i0, i1): from their screen gradient
// (n x 9) to the parameter gradients in the planar layout of the parameters
// (means [3][n_pad], log_scales [3][n_pad], quats [4][n_pad], opacity_logits
// [n_pad], sh [3][K][n_pad]); writes those Gaussians' entries only (a culled
// Gaussian or one with a zero screen gradient gets zeros). Any output may be null.
void or_project_backward(void* h, const double* screen_grad, int64_t i0, int64_t i1,
                         double* g_means, double* g_ls, double* g_quats, double* g_logits,
                         double* g_sh) {
  const Ctx& c = *static_cast<Ctx*>(h);
  const int64_t n = c.n, np = c.n_pad;
  const int K = (c.sh_degree + 1) * (c.sh_degree + 1);
  const int nk = (c.active_degree + 1) * (c.active_degree + 1);
  i0 = std::max<int64_t>(i0, 0);
  i1 = std::min<int64_t>(i1, n);
  for (int64_t i = i0; i < i1; ++i) {
    if (g_means)
      for (int j = 0; j < 3; ++j) g_means[j * np + i] = 0.0;
    if (g_ls)
      for (int j = 0; j < 3; ++j) g_ls[j * np + i] = 0.0;
    if (g_quats)
      for (int j = 0; j < 4; ++j) g_quats[j * np + i] = 0.0;
    if (g_logits) g_logits[i] = 0.0;
    if (g_sh)
      for (int k = 0; k < 3 * K; ++k) g_sh[static_cast<size_t>(k) * np + i] = 0.0;
    if (c.aux[i].touched == 0) continue;
    const double* gs = &screen_grad[static_cast<size_t>(i) * kScreen];
    bool any = false;
    for (int o = 0; o < kScreen; ++o) any = any || gs[o] != 0.0;
    if (!any) continue;  // a zero screen gradient has a zero parameter gradient
    // Jacobian of the screen state w.r.t. (mean 3, log-scale 3, quat 4, logit).
    using D = Dual<11>;
    D p[3] = {seed<11>(c.means[i], 0), seed<11>(c.means[np + i], 1),
              seed<11>(c.means[2 * np + i], 2)};
    D ls[3] = {seed<11>(c.ls[i], 3), seed<11>(c.ls[np + i], 4), seed<11>(c.ls[2 * np + i], 5)};
    D q[4] = {seed<11>(c.quats[i], 6), seed<11>(c.quats[np + i], 7),
              seed<11>(c.quats[2 * np + i], 8), seed<11>(c.quats[3 * np + i], 9)};
    D logit = seed<11>(c.logits[i], 10);
    Proj<D> P;
    Aux X;
    project<D>(c.cam, p, ls, q, logit, &c.sh[i], np, c.active_degree, P, X, c.opacity_rect,
               c.mip_comp);
    const D* outs[kScreen] = {&P.u, &P.v, &P.A, &P.B, &P.C, &P.o, &P.rgb[0], &P.rgb[1], &P.rgb[2]};
    double gp[11] = {0};
    for (int o = 0; o < kScreen; ++o)
      for (int j = 0; j < 11; ++j) gp[j] += gs[o] * outs[o]->d[j];
    if (g_means)
      for (int j = 0; j < 3; ++j) g_means[j * np + i] = gp[j];
    if (g_ls)
      for (int j = 0; j < 3; ++j) g_ls[j * np + i] = gp[3 + j];
    if (g_quats)
      for (int j = 0; j < 4; ++j) g_quats[j * np + i] = gp[6 + j];
    if (g_logits) g_logits[i] = gp[10];
    // The colour is linear in its SH coefficients: dc/dsh_k = Y_k (zero if clamped).
    if (g_sh)
      for (int ch = 0; ch < 3; ++ch) {
        if (X.clamped[ch]) continue;
        for (int k = 0; k < nk; ++k)
          g_sh[(static_cast<size_t>(ch) * K + k) * np + i] = gs[6 + ch] * X.Y[k];
      }
  }
}

// Gradient of the loss with respect to the camera pose ("How a computer
// rebuilds a real place ... Gaussian Splats", section "Forgiving the camera
// and the light": the render depends on the camera, so backprop gives it a
// gradient too). The pose moves as R <- exp([w]x) R, t <- t + dt: a rotation
// w of the camera frame and a shift dt of the translation, the
// parametrisation of that section's code (rotation blame = cross(p_c - t,
// dL/dp_c), translation blame = dL/dp_c). Here the derivative is the exact
// one, by dual numbers through the whole projection: besides the position
// path it includes the rotation of each Gaussian's camera-space covariance
// and the move of the camera centre campos = -R^T t in the view direction of
// the colour. out = {dL/dw (3), dL/dt (3)}, summed over the Gaussians from
// their screen gradient (n x 9).
void or_camera_backward(void* h, const double* screen_grad, double* out) {
  const Ctx& c = *static_cast<Ctx*>(h);
  using D = Dual<6>;
  PoseCamera<D> pc;
  pc.width = c.cam.width;
  pc.height = c.cam.height;
  pc.fx = c.cam.fx;
  pc.fy = c.cam.fy;
  pc.cx = c.cam.cx;
  pc.cy = c.cam.cy;
  pc.near_z = c.cam.near_z;
  const D w[3] = {seed<6>(0.0, 0), seed<6>(0.0, 1), seed<6>(0.0, 2)};
  // exp([w]x) = I + [w]x + O(w^2): the first-order part gives the exact derivative at w = 0
  const D Wx[9] = {D(0.0), -w[2], w[1], w[2], D(0.0), -w[0], -w[1], w[0], D(0.0)};
  for (int r = 0; r < 3; ++r)
    for (int col = 0; col < 3; ++col) {
      D acc(c.cam.R[3 * r + col]);
      for (int k = 0; k < 3; ++k) acc = acc + Wx[3 * r + k] * c.cam.R[3 * k + col];
      pc.R[3 * r + col] = acc;
    }
  for (int i = 0; i < 3; ++i) pc.t[i] = c.cam.t[i] + seed<6>(0.0, 3 + i);
  // campos = -R^T t as a function of the pose; its value stays the camera's own
  for (int i = 0; i < 3; ++i) {
    D acc(0.0);
    for (int k = 0; k < 3; ++k) acc = acc + pc.R[3 * k + i] * pc.t[k];
    pc.campos[i] = -acc;
    pc.campos[i].v = c.cam.campos[i];
  }
  const int64_t np = c.n_pad;
  double g[6] = {0, 0, 0, 0, 0, 0};
  for (int64_t i = 0; i < c.n; ++i) {
    if (c.aux[i].touched == 0) continue;
    const double* gs = &screen_grad[static_cast<size_t>(i) * kScreen];
    bool any = false;
    for (int o = 0; o < kScreen; ++o) any = any || gs[o] != 0.0;
    if (!any) continue;
    const D p[3] = {D(c.means[i]), D(c.means[np + i]), D(c.means[2 * np + i])};
    const D ls[3] = {D(c.ls[i]), D(c.ls[np + i]), D(c.ls[2 * np + i])};
    const D q[4] = {D(c.quats[i]), D(c.quats[np + i]), D(c.quats[2 * np + i]), D(c.quats[3 * np + i])};
    const D logit(c.logits[i]);
    Proj<D> P;
    Aux X;
    if (!project<D>(pc, p, ls, q, logit, &c.sh[i], np, c.active_degree, P, X, c.opacity_rect,
                    c.mip_comp))
      continue;
    const D* outs[kScreen] = {&P.u, &P.v, &P.A, &P.B, &P.C, &P.o, &P.rgb[0], &P.rgb[1], &P.rgb[2]};
    for (int o = 0; o < kScreen; ++o)
      for (int j = 0; j < 6; ++j) g[j] += gs[o] * outs[o]->d[j];
  }
  for (int j = 0; j < 6; ++j) out[j] = g[j];
}

// Backward from dL/dimage [3][H][W] over the pixel rows [y0, y1) (other rows
// contribute nothing): the screen gradient n x 9 and the parameter gradients of
// all Gaussians (padding entries of the planar outputs are zeroed). Any output
// pointer may be null.
void or_backward_rows(void* h, int32_t y0, int32_t y1, const double* dimage, double* screen_grad,
                      double* g_means, double* g_ls, double* g_quats, double* g_logits,
                      double* g_sh) {
  const Ctx& c = *static_cast<Ctx*>(h);
  const int64_t n = c.n, np = c.n_pad;
  std::vector<double> sg(static_cast<size_t>(n) * kScreen, 0.0);
  or_blend_backward_rows(h, y0, y1, dimage, sg.data());
  if (screen_grad) std::memcpy(screen_grad, sg.data(), sg.size() * sizeof(double));
  const int K = (c.sh_degree + 1) * (c.sh_degree + 1);
  if (g_means) std::memset(g_means, 0, sizeof(double) * 3 * np);
  if (g_ls) std::memset(g_ls, 0, sizeof(double) * 3 * np);
  if (g_quats) std::memset(g_quats, 0, sizeof(double) * 4 * np);
  if (g_logits) std::memset(g_logits, 0, sizeof(double) * np);
  if (g_sh) std::memset(g_sh, 0, sizeof(double) * 3 * K * np);
  or_project_backward(h, sg.data(), 0, n, g_means, g_ls, g_quats, g_logits, g_sh);
}

void or_backward(void* h, const double* dimage, double* screen_grad, double* g_means,
                 double* g_ls, double* g_quats, double* g_logits, double* g_sh) {
  or_backward_rows(h, 0, static_cast<Ctx*>(h)->cam.height, dimage, screen_grad, g_means, g_ls,
                   g_quats, g_logits, g_sh);
}

// ------------------------------------------------------------------- loss --
// (1 - lambda) L1 + lambda (1 - SSIM) of image x against target y, both
// [3][H][W] float32. out3 = {loss, L1, SSIM}; dimage = dL/dx (may be null).
}  // extern "C"

namespace {

template <class In>
int loss_impl(int32_t H, int32_t W, const In* x, const In* y, double lambda, double* out3,
              double* dimage) {
  if (H <= 0 || W <= 0) return 1;
  const double C1 = 0.01 * 0.01, C2 = 0.03 * 0.03;
  const int R = 5;
  double g1[11], gsum = 0.0;
  for (int i = -R; i <= R; ++i) gsum += (g1[i + R] = std::exp(-(i * i) / (2.0 * 1.5 * 1.5)));
  for (double& w : g1) w /= gsum;
  auto w2 = [&](int di, int dj) { return g1[di + R] * g1[dj + R]; };

  const size_t HW = static_cast<size_t>(H) * W;
  const double inv = 1.0 / (3.0 * static_cast<double>(HW));
  double l1 = 0.0, ssim = 0.0;
  // Per-map partial derivatives dS/d(mu_x), dS/d(E[x^2]), dS/d(E[xy]).
  std::vector<double> dmu(HW), dxx(HW), dxy(HW);
  for (int ch = 0; ch < 3; ++ch) {
    const In* X = x + ch * HW;
    const In* Yv = y + ch * HW;
    for (int i = 0; i < H; ++i)
      for (int j = 0; j < W; ++j) {
        double mx = 0, my = 0, exx = 0, eyy = 0, exy = 0;
        for (int di = -R; di <= R; ++di)
          for (int dj = -R; dj <= R; ++dj) {
            int ii = i + di, jj = j + dj;
            if (ii < 0 || ii >= H || jj < 0 || jj >= W) continue;  // zero padding
            double w = w2(di, dj);
            double xv = X[ii * W + jj], yv = Yv[ii * W + jj];
            mx += w * xv;
            my += w * yv;
            exx += w * xv * xv;
            eyy += w * yv * yv;
            exy += w * xv * yv;
          }
        Dual<3> Mx = seed<3>(mx, 0), Exx = seed<3>(exx, 1), Exy = seed<3>(exy, 2);
        Dual<3> sx2 = Exx - Mx * Mx;
        double sy2 = eyy - my * my;
        Dual<3> sxy = Exy - Mx * my;
        Dual<3> S = ((2.0 * Mx * my + C1) * (2.0 * sxy + C2)) /
                    ((Mx * Mx + my * my + C1) * (sx2 + sy2 + C2));
        ssim += S.v;
        size_t p = static_cast<size_t>(i) * W + j;
        dmu[p] = S.d[0];
        dxx[p] = S.d[1];
        dxy[p] = S.d[2];
        double r = static_cast<double>(X[p]) - static_cast<double>(Yv[p]);
        l1 += std::fabs(r);
      }
    if (dimage) {
      for (int i = 0; i < H; ++i)
        for (int j = 0; j < W; ++j) {
          size_t p = static_cast<size_t>(i) * W + j;
          double xv = X[p], yv = Yv[p];
          double acc = 0.0;
          for (int di = -R; di <= R; ++di)
            for (int dj = -R; dj <= R; ++dj) {
              int ii = i + di, jj = j + dj;
              if (ii < 0 || ii >= H || jj < 0 || jj >= W) continue;
              size_t q = static_cast<size_t>(ii) * W + jj;
              acc += w2(di, dj) * (dmu[q] + 2.0 * xv * dxx[q] + yv * dxy[q]);
            }
          double r = xv - yv;
          double sgn = r > 0 ? 1.0 : (r < 0 ? -1.0 : 0.0);
          dimage[ch * HW + p] = (1.0 - lambda) * sgn * inv - lambda * inv * acc;
        }
    }
  }
  l1 *= inv;
  ssim *= inv;
  out3[0] = (1.0 - lambda) * l1 + lambda * (1.0 - ssim);
  out3[1] = l1;
  out3[2] = ssim;
  return 0;
}

}  // namespace

extern "C" {

int or_loss(int32_t H, int32_t W, const float* x, const float* y, double lambda, double* out3,
            double* dimage) {
  return loss_impl<float>(H, W, x, y, lambda, out3, dimage);
}

// The same loss on float64 images (used by the central-difference checks).
int or_loss_f64(int32_t H, int32_t W, const double* x, const double* y, double lambda,
                double* out3, double* dimage) {
  return loss_impl<double>(H, W, x, y, lambda, out3, dimage);
}

// ------------------------------------------------------------------- Adam --
// One Adam step at step number t >= 1 on float64 arrays; zeroes the gradient.
void or_adam(int64_t count, double* p, double* g, double* m, double* v, double lr, double beta1,
             double beta2, double eps, int32_t t) {
  for (int64_t i = 0; i < count; ++i) {
    m[i] = beta1 * m[i] + (1.0 - beta1) * g[i];
    v[i] = beta2 * v[i] + (1.0 - beta2) * g[i] * g[i];
    double mh = m[i] / (1.0 - std::pow(beta1, t));
    double vh = v[i] / (1.0 - std::pow(beta2, t));
    p[i] = p[i] - lr * mh / (std::sqrt(vh) + eps);
    g[i] = 0.0;
  }
}

// ------------------------------------------------------- small test entries --
// Blend one pixel (px, py) over screen-space Gaussians given as n x 9
// (u, v, A, B, C, o, r, g, b), visited in the given order, with no tiling.
// Returns colour and final T; if dldI is given, also the screen gradient
// n x 9 of sum_c dldI[c] I[c].
void or_blend_screen(int32_t n, const double* screen, int32_t norder, const int32_t* order,
                     double px, double py, const double* bg, const double* dldI, double* rgb,
                     double* T_out, double* sgrad) {
  Ctx c;
  c.cam.bg[0] = bg[0];
  c.cam.bg[1] = bg[1];
  c.cam.bg[2] = bg[2];
  c.cam.width = 1;
  c.cam.height = 1;
  c.screen.assign(screen, screen + static_cast<size_t>(n) * kScreen);
  // Pixel (px, py) is mapped to (0, 0) of a one-tile image by shifting centres.
  for (int32_t i = 0; i < n; ++i) {
    c.screen[kScreen * i + 0] -= px;
    c.screen[kScreen * i + 1] -= py;
  }
  for (int32_t k = 0; k < norder; ++k) c.entries.push_back({0, 0u, order[k]});
  c.range_lo.assign(1, 0);
  c.range_hi.assign(1, norder);
  PixelResult r;
  std::vector<Contribution> list;
  walk_pixel(c, 0, 0, r, &list);
  for (int ch = 0; ch < 3; ++ch) rgb[ch] = r.rgb[ch];
  *T_out = r.T;
  if (dldI && sgrad) {
    std::memset(sgrad, 0, sizeof(double) * kScreen * n);
    backward_pixel(c, list, dldI, sgrad);
  }
}

// Real SH basis values (k < (degree+1)^2, basis 1 at k = 0) at unit directions
// dirs n x 3; out n x 16.
void or_sh_basis(int32_t degree, int64_t n, const double* dirs, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    double Y[16] = {0};
    sh_basis().eval(degree, dirs[3 * i], dirs[3 * i + 1], dirs[3 * i + 2], Y);
    for (int k = 0; k < 16; ++k) out[16 * i + k] = Y[k];
  }
}

// Rotation matrix (row-major) of q / |q| and the 3D covariance R S S^T R^T.
void or_rotation_cov(const double* q, const double* ls, double* R, double* Sigma) {
  double qn = std::sqrt(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
  double qh[4] = {q[0] / qn, q[1] / qn, q[2] / qn, q[3] / qn};
  quat_to_rot(qh, R);
  covariance3d(ls, q, Sigma);
}

}  // extern "C"
