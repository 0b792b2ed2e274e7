"""Seeded synthetic scenes and cameras shared by the CUDA path and the oracle.

This module only draws random numbers and builds camera poses; it holds none of
the rasteriser's arithmetic (no projection, blending, loss or gradient), so the
tests can feed the very same inputs to both implementations.

Scene shapes follow the workloads the pages describe: Gaussians with log-scales,
quaternions, opacity logits and spherical-harmonic colour coefficients
("Gaussian splatting training" study notes, slide "The stored scales are
log-scales and the stored opacity is a logit"), viewed by posed pinhole cameras
("How a computer rebuilds a real place ... Gaussian Splats", section
"Flattening a 3D blob into a 2D oval (EWA projection)").

Parameter layout (structure of arrays, planar float32, N padded to a multiple
of 4 so every plane starts on a 16-byte boundary):

    means           [3][n_pad]
    log_scales      [3][n_pad]
    quats           [4][n_pad]      (w, x, y, z), not necessarily unit length
    opacity_logits  [n_pad]
    sh              [3][K][n_pad]   K = (sh_degree + 1)**2, k = 0 is the base RGB

Padding entries (index >= n) are zero and are never read by the rasteriser.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass
class Camera:
    """A pinhole camera. Pixel (i, j) sits at continuous coordinate (i, j);
    camera axes are x right, y down, z forward; p_cam = R @ p_world + t."""

    width: int
    height: int
    fx: float
    fy: float
    cx: float
    cy: float
    R: np.ndarray  # (3, 3) float32, rows are the camera axes in world space
    t: np.ndarray  # (3,) float32
    campos: np.ndarray  # (3,) float32, camera centre in world space
    bg: np.ndarray  # (3,) float32 background colour
    near_z: float = 0.2


@dataclasses.dataclass
class Scene:
    n: int
    n_pad: int
    sh_degree: int
    means: np.ndarray
    log_scales: np.ndarray
    quats: np.ndarray
    opacity_logits: np.ndarray
    sh: np.ndarray
    cameras: list
    name: str = ""

    @property
    def sh_k(self) -> int:
        return (self.sh_degree + 1) ** 2

    def groups(self) -> dict:
        return {
            "means": self.means,
            "log_scales": self.log_scales,
            "quats": self.quats,
            "opacity_logits": self.opacity_logits,
            "sh": self.sh,
        }

    def copy(self) -> "Scene":
        return dataclasses.replace(
            self,
            means=self.means.copy(),
            log_scales=self.log_scales.copy(),
            quats=self.quats.copy(),
            opacity_logits=self.opacity_logits.copy(),
            sh=self.sh.copy(),
            cameras=list(self.cameras),
        )


GROUP_NAMES = ("means", "log_scales", "quats", "opacity_logits", "sh")


def pad4(n: int) -> int:
    return max(4, (n + 3) // 4 * 4)


def look_at(pos, target, width, height, f, bg=(0.0, 0.0, 0.0), near_z=0.2) -> Camera:
    """Camera at `pos` looking at `target` with world +y as the up hint.

    z_c = normalize(target - pos); x_c = normalize(z_c x (0, 1, 0));
    y_c = z_c x x_c; rows of R = (x_c, y_c, z_c); t = -R pos; c = (W/2, H/2).
    """
    pos = np.asarray(pos, dtype=np.float64)
    target = np.asarray(target, dtype=np.float64)
    z = target - pos
    z /= np.linalg.norm(z)
    x = np.cross(z, np.array([0.0, 1.0, 0.0]))
    x /= np.linalg.norm(x)
    y = np.cross(z, x)
    R = np.stack([x, y, z]).astype(np.float32)
    t = (-(R.astype(np.float64) @ pos)).astype(np.float32)
    return Camera(
        width=int(width), height=int(height),
        fx=float(np.float32(f)), fy=float(np.float32(f)),
        cx=float(np.float32(width / 2.0)), cy=float(np.float32(height / 2.0)),
        R=R, t=t, campos=pos.astype(np.float32),
        bg=np.asarray(bg, dtype=np.float32), near_z=float(np.float32(near_z)),
    )


def identity_camera(width, height, f, bg=(0.0, 0.0, 0.0)) -> Camera:
    return Camera(
        width=int(width), height=int(height),
        fx=float(np.float32(f)), fy=float(np.float32(f)),
        cx=float(np.float32(width / 2.0)), cy=float(np.float32(height / 2.0)),
        R=np.eye(3, dtype=np.float32), t=np.zeros(3, np.float32),
        campos=np.zeros(3, np.float32), bg=np.asarray(bg, dtype=np.float32),
    )


def ring_cameras(n_cams, radius, width, height, f) -> list:
    """n_cams cameras on a circle of `radius` in the y = 0 plane, angles 2*pi*k/n,
    all looking at the origin."""
    cams = []
    for k in range(n_cams):
        a = 2.0 * math.pi * k / n_cams
        cams.append(look_at((radius * math.cos(a), 0.0, radius * math.sin(a)),
                            (0.0, 0.0, 0.0), width, height, f))
    return cams


def _empty(n, sh_degree, dtype=np.float32):
    n_pad = pad4(n)
    K = (sh_degree + 1) ** 2
    return (n_pad,
            np.zeros((3, n_pad), dtype), np.zeros((3, n_pad), dtype),
            np.zeros((4, n_pad), dtype), np.zeros((n_pad,), dtype),
            np.zeros((3, K, n_pad), dtype))


def _unit_quats(rng, n):
    q = rng.standard_normal((4, n))
    return q / np.linalg.norm(q, axis=0, keepdims=True)


def _sh_coeffs(rng, sh, n, dc_rgb_uniform=True, hi_sigma=0.1):
    K = sh.shape[1]
    sh[:, 0, :n] = rng.uniform(0.0, 1.0, (3, n))
    if K > 1:
        sh[:, 1:, :n] = rng.normal(0.0, hi_sigma, (3, K - 1, n))


def make_scene(name, means, log_scales, quats, logits, sh_degree, sh_fill, cameras,
               dtype=np.float32) -> Scene:
    """Packs per-Gaussian arrays into the padded planar layout. float64 scenes are
    only for the oracle's own checks; the CUDA path takes float32."""
    n = means.shape[1]
    n_pad, M, LS, Q, O, SH = _empty(n, sh_degree, dtype)
    M[:, :n] = means
    LS[:, :n] = log_scales
    Q[:, :n] = quats
    O[:n] = logits
    SH[:, :, :n] = sh_fill
    return Scene(n=n, n_pad=n_pad, sh_degree=sh_degree, means=M, log_scales=LS,
                 quats=Q, opacity_logits=O, sh=SH, cameras=cameras, name=name)


def tiny(seed=0) -> Scene:
    """64 Gaussians, one 64x64 camera (f = 64, c = 32, identity pose), SH degree 0."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 64
    xy = rng.uniform(-1.0, 1.0, (2, n))
    z = rng.uniform(2.0, 6.0, (1, n))
    means = np.concatenate([xy, z])
    ls = rng.normal(math.log(0.08), 0.3, (3, n))
    q = _unit_quats(rng, n)
    logits = rng.normal(0.0, 1.0, n)
    sh = rng.uniform(0.0, 1.0, (3, 1, n))
    return make_scene("tiny", means, ls, q, logits, 0, sh, [identity_camera(64, 64, 64.0)])


def small(seed=0) -> Scene:
    """10k Gaussians on a shell of radius N(1, 0.1^2), SH degree 3, one 256^2 camera
    at (0, 0, -3) looking at the origin. Log-scales are drawn per axis."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 10_000
    d = rng.standard_normal((3, n))
    d /= np.linalg.norm(d, axis=0, keepdims=True)
    r = rng.normal(1.0, 0.1, n)
    means = d * r
    ls = rng.normal(math.log(0.02), 0.5, (3, n))
    q = _unit_quats(rng, n)
    logits = rng.normal(0.0, 1.5, n)
    sh = np.zeros((3, 16, n))
    sh[:, 0] = rng.uniform(0.0, 1.0, (3, n))
    sh[:, 1:] = rng.normal(0.0, 0.1, (3, 15, n))
    cam = look_at((0.0, 0.0, -3.0), (0.0, 0.0, 0.0), 256, 256, 256.0)
    return make_scene("small", means, ls, q, logits, 3, sh, [cam])


def mid(seed=0) -> Scene:
    """500k Gaussians uniform in [-5, 5]^3, anisotropic log-scales N(log 0.01, 0.7^2),
    SH degree 3, opacity logits N(-1, 2^2); 16 ring cameras (r = 15) at 1280x720, f = 1100."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n = 500_000
    means = rng.uniform(-5.0, 5.0, (3, n))
    ls = rng.normal(math.log(0.01), 0.7, (3, n))
    q = _unit_quats(rng, n)
    logits = rng.normal(-1.0, 2.0, n)
    sh = np.zeros((3, 16, n), np.float32)
    sh[:, 0] = rng.uniform(0.0, 1.0, (3, n))
    sh[:, 1:] = rng.normal(0.0, 0.1, (3, 15, n))
    return make_scene("mid", means, ls, q, logits, 3, sh,
                      ring_cameras(16, 15.0, 1280, 720, 1100.0))


def dense(seed=0, n=3_000_000) -> Scene:
    """3M Gaussians drawn from 64 clusters (centres U[-3, 3]^3, members N(centre, 0.3^2)),
    log-scales N(log 0.005, 0.6^2) per axis, SH degree 3, opacity logits N(0, 2^2);
    32 ring cameras (r = 10) at 1920x1080, f = 1600."""
    rng = np.random.Generator(np.random.PCG64(seed))
    centres = rng.uniform(-3.0, 3.0, (3, 64))
    member = rng.integers(0, 64, n)
    means = centres[:, member] + rng.normal(0.0, 0.3, (3, n))
    ls = rng.normal(math.log(0.005), 0.6, (3, n))
    q = _unit_quats(rng, n)
    logits = rng.normal(0.0, 2.0, n)
    sh = np.zeros((3, 16, n), np.float32)
    sh[:, 0] = rng.uniform(0.0, 1.0, (3, n))
    sh[:, 1:] = rng.normal(0.0, 0.1, (3, 15, n))
    return make_scene("dense", means, ls, q, logits, 3, sh,
                      ring_cameras(32, 10.0, 1920, 1080, 1600.0))


def heavy_tail(seed=0, n=6_000_000) -> Scene:
    """6M Gaussians uniform in [-20, 20] x [-5, 5] x [-20, 20]; log-scales per axis from
    0.9 N(log 0.004, 0.4^2) + 0.1 N(log 0.2, 0.5^2); SH degree 3; logits N(0, 2^2);
    32 ring cameras (r = 35) at 1920x1080, f = 1600."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lo = np.array([[-20.0], [-5.0], [-20.0]])
    hi = np.array([[20.0], [5.0], [20.0]])
    means = rng.uniform(lo, hi, (3, n))
    big = rng.uniform(0.0, 1.0, n) < 0.1
    ls = np.where(big[None, :], rng.normal(math.log(0.2), 0.5, (3, n)),
                  rng.normal(math.log(0.004), 0.4, (3, n)))
    q = _unit_quats(rng, n)
    logits = rng.normal(0.0, 2.0, n)
    sh = np.zeros((3, 16, n), np.float32)
    sh[:, 0] = rng.uniform(0.0, 1.0, (3, n))
    sh[:, 1:] = rng.normal(0.0, 0.1, (3, 15, n))
    return make_scene("heavy_tail", means, ls, q, logits, 3, sh,
                      ring_cameras(32, 35.0, 1920, 1080, 1600.0))


CONFIGS = {"tiny": tiny, "small": small, "mid": mid, "dense": dense, "heavy_tail": heavy_tail}


def perturbed(scene: Scene, sigma=0.05, seed=1) -> Scene:
    """A copy with N(0, sigma^2) added to every stored scalar of every real Gaussian."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = scene.copy()
    n = scene.n
    for name in GROUP_NAMES:
        arr = getattr(out, name)
        view = arr[..., :n]
        view += rng.normal(0.0, sigma, view.shape).astype(np.float32)
    return out


def uniform_image(height, width, seed=2) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.uniform(0.0, 1.0, (3, height, width)).astype(np.float32)


def camera_schedule(n_cams, n_iters, seed=0) -> np.ndarray:
    """Camera index per iteration: concatenated seeded permutations of range(n_cams)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    while len(out) < n_iters:
        out.extend(rng.permutation(n_cams).tolist())
    return np.asarray(out[:n_iters], dtype=np.int64)


def random_screen_gaussians(n, width, height, seed=3, scale=(1.0, 6.0)):
    """Screen-space Gaussians (u, v, A, B, C, o, r, g, b) for blend-only tests:
    centres uniform over the image, a positive-definite conic drawn directly as
    A = 1/s1^2, C = 1/s2^2, B = rho sqrt(A C) with s in the given pixel range and
    |rho| < 0.8, opacity U[0.05, 0.95], colour U[0, 1]. Returns (n, 9) float64
    together with per-Gaussian depths U[1, 10]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.uniform(0, width - 1, n)
    v = rng.uniform(0, height - 1, n)
    s1 = rng.uniform(*scale, n)
    s2 = rng.uniform(*scale, n)
    rho = rng.uniform(-0.8, 0.8, n)
    A = 1.0 / s1 ** 2
    C = 1.0 / s2 ** 2
    B = rho * np.sqrt(A * C)
    o = rng.uniform(0.05, 0.95, n)
    rgb = rng.uniform(0.0, 1.0, (n, 3))
    depth = rng.uniform(1.0, 10.0, n)
    return np.column_stack([u, v, A, B, C, o, rgb]), depth
