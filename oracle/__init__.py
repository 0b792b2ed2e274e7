"""ctypes front end of the float64 CPU oracle (test infrastructure only).

Only the tests, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package. It never imports the CUDA package and the
CUDA package never imports it; both take their inputs from the seeded scene
generator.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


class OrCamera(ctypes.Structure):
    _fields_ = [
        ("width", ctypes.c_int32), ("height", ctypes.c_int32),
        ("fx", ctypes.c_double), ("fy", ctypes.c_double),
        ("cx", ctypes.c_double), ("cy", ctypes.c_double),
        ("R", ctypes.c_double * 9), ("t", ctypes.c_double * 3),
        ("campos", ctypes.c_double * 3), ("bg", ctypes.c_double * 3),
        ("near_z", ctypes.c_double),
    ]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.or_create.restype = P
        L.or_destroy.argtypes = [P]
        L.or_set_scene.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                   P, P, P, P, P, ctypes.POINTER(OrCamera)]
        L.or_set_scene.restype = ctypes.c_int
        L.or_set_scene_f64.argtypes = L.or_set_scene.argtypes
        L.or_set_scene_f64.restype = ctypes.c_int
        L.or_get_preprocess.argtypes = [P] * 9
        L.or_num_entries.argtypes = [P]
        L.or_num_entries.restype = ctypes.c_int64
        L.or_get_sorted.argtypes = [P] * 4
        L.or_render.argtypes = [P] * 6
        L.or_render_pixels.argtypes = [P, ctypes.c_int64] + [P] * 6
        L.or_render_rows.argtypes = [P, ctypes.c_int32, ctypes.c_int32] + [P] * 5
        L.or_backward_rows.argtypes = [P, ctypes.c_int32, ctypes.c_int32] + [P] * 7
        L.or_backward.argtypes = [P] * 8
        L.or_blend_backward_rows.argtypes = [P, ctypes.c_int32, ctypes.c_int32, P, P]
        L.or_set_option.argtypes = [P, ctypes.c_int32, ctypes.c_int32]
        L.or_set_option.restype = ctypes.c_int
        L.or_project_backward.argtypes = [P, P, ctypes.c_int64, ctypes.c_int64] + [P] * 5
        L.or_loss.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_double, P, P]
        L.or_loss.restype = ctypes.c_int
        L.or_loss_f64.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_double, P, P]
        L.or_loss_f64.restype = ctypes.c_int
        L.or_adam.argtypes = [ctypes.c_int64, P, P, P, P, ctypes.c_double, ctypes.c_double,
                              ctypes.c_double, ctypes.c_double, ctypes.c_int32]
        L.or_blend_screen.argtypes = [ctypes.c_int32, P, ctypes.c_int32, P, ctypes.c_double,
                                      ctypes.c_double, P, P, P, P, P]
        L.or_sh_basis.argtypes = [ctypes.c_int32, ctypes.c_int64, P, P]
        L.or_rotation_cov.argtypes = [P, P, P, P]
        L.or_camera_backward.argtypes = [P, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def camera(cam, f64=False) -> OrCamera:
    """The camera as the oracle reads it: the float32 values the CUDA path
    receives, widened to float64; with f64 the camera's own values unrounded
    (for derivative checks that move the pose by less than a float32 step)."""
    rnd = (lambda v: float(v)) if f64 else (lambda v: float(np.float32(v)))
    c = OrCamera()
    c.width, c.height = int(cam.width), int(cam.height)
    c.fx, c.fy, c.cx, c.cy = (rnd(v) for v in (cam.fx, cam.fy, cam.cx, cam.cy))
    for i, v in enumerate(np.asarray(cam.R, np.float64).reshape(-1)):
        c.R[i] = rnd(v)
    for name in ("t", "campos", "bg"):
        arr = getattr(c, name)
        for i, v in enumerate(np.asarray(getattr(cam, name), np.float64).reshape(-1)):
            arr[i] = rnd(v)
    c.near_z = rnd(cam.near_z)
    return c


class Oracle:
    """One scene seen by one camera: preprocess and tile lists are built on
    construction; render/backward walk the lists per pixel."""

    def __init__(self, scene, cam, active_degree=None, opacity_rect=False, camera_f64=False, mip_comp=False):
        self.L = lib()
        self.scene = scene
        self.cam = cam
        self.h = self.L.or_create()
        if opacity_rect:
            self.L.or_set_option(self.h, 1, 1)
        if mip_comp:  # opacity times the Mip-Splatting compensation factor
            self.L.or_set_option(self.h, 2, 1)
        self.active_degree = scene.sh_degree if active_degree is None else active_degree
        f64 = np.asarray(scene.means).dtype == np.float64
        dt = np.float64 if f64 else np.float32
        arrs = [np.ascontiguousarray(a, dtype=dt) for a in
                (scene.means, scene.log_scales, scene.quats, scene.opacity_logits, scene.sh)]
        self._keep = arrs
        self._cam = camera(cam, camera_f64)
        fn = self.L.or_set_scene_f64 if f64 else self.L.or_set_scene
        rc = fn(self.h, scene.n, scene.n_pad, scene.sh_degree, self.active_degree,
                *[_p(a) for a in arrs], ctypes.byref(self._cam))
        if rc != 0:
            raise ValueError("oracle rejected the scene")

    def __del__(self):
        h = getattr(self, "h", None)
        if h:
            self.L.or_destroy(h)
            self.h = None

    @property
    def tiles(self):
        return ((self.cam.width + 15) // 16, (self.cam.height + 15) // 16)

    def preprocess(self) -> dict:
        n = self.scene.n
        out = dict(screen=np.zeros((n, 9)), cov2d=np.zeros((n, 3)), depth=np.zeros(n),
                   depth_key=np.zeros(n, np.float32), radius=np.zeros(n),
                   rect=np.zeros((n, 4), np.int32), touched=np.zeros(n, np.int32),
                   clamped=np.zeros((n, 3), np.uint8))
        self.L.or_get_preprocess(self.h, *[_p(out[k]) for k in
                                           ("screen", "cov2d", "depth", "depth_key", "radius",
                                            "rect", "touched", "clamped")])
        return out

    def sorted(self) -> dict:
        k = self.L.or_num_entries(self.h)
        tx, ty = self.tiles
        ids = np.zeros(k, np.int32)
        tiles = np.zeros(k, np.int32)
        ranges = np.zeros((tx * ty, 2), np.int64)
        self.L.or_get_sorted(self.h, _p(ids), _p(tiles), _p(ranges))
        return dict(ids=ids, tiles=tiles, ranges=ranges)

    def render(self) -> dict:
        H, W = self.cam.height, self.cam.width
        out = dict(image=np.zeros((3, H, W)), final_T=np.zeros((H, W)),
                   n_contrib=np.zeros((H, W), np.int32), ambiguous=np.zeros((H, W), np.uint8),
                   stats=np.zeros(2, np.int64))
        self.L.or_render(self.h, *[_p(out[k]) for k in
                                   ("image", "final_T", "n_contrib", "ambiguous", "stats")])
        return out

    def render_pixels(self, px, py) -> dict:
        px = np.ascontiguousarray(px, np.int32)
        py = np.ascontiguousarray(py, np.int32)
        n = px.size
        out = dict(rgb=np.zeros((n, 3)), T=np.zeros(n), n_contrib=np.zeros(n, np.int32),
                   ambiguous=np.zeros(n, np.uint8))
        self.L.or_render_pixels(self.h, n, _p(px), _p(py), _p(out["rgb"]), _p(out["T"]),
                                _p(out["n_contrib"]), _p(out["ambiguous"]))
        return out

    def replay_pixels(self, px, py, flip) -> dict:
        """The forward at pixels (px, py) with, per pixel, the near-threshold
        decisions selected by bit mask `flip` taken the other way (bit k = the
        k-th decision within the ambiguity margin, in walk order); n_amb = the
        number of such decisions the walk met. flip = 0 is the plain walk."""
        px = np.ascontiguousarray(px, np.int32)
        py = np.ascontiguousarray(py, np.int32)
        flip = np.ascontiguousarray(np.broadcast_to(np.asarray(flip, np.uint32), px.shape))
        n = px.size
        out = dict(rgb=np.zeros((n, 3)), T=np.zeros(n), n_contrib=np.zeros(n, np.int32),
                   n_amb=np.zeros(n, np.int32))
        self.L.or_render_pixels_replay(self.h, n, _p(px), _p(py), _p(flip), _p(out["rgb"]), _p(out["T"]),
                                       _p(out["n_contrib"]), _p(out["n_amb"]))
        return out

    def render_rows(self, y0, y1, out=None) -> dict:
        """Forward over the pixel rows [y0, y1) into full-size outputs (`out`, as
        returned by an earlier call, is reused when given)."""
        H, W = self.cam.height, self.cam.width
        if out is None:
            out = dict(image=np.zeros((3, H, W)), final_T=np.zeros((H, W)),
                       n_contrib=np.zeros((H, W), np.int32), ambiguous=np.zeros((H, W), np.uint8),
                       stats=np.zeros(2, np.int64))
        self.L.or_render_rows(self.h, int(y0), int(y1), *[_p(out[k]) for k in
                                                           ("image", "final_T", "n_contrib",
                                                            "ambiguous", "stats")])
        return out

    def backward(self, dimage, rows=None) -> dict:
        """Parameter and screen gradients from dL/dimage; `rows` = (y0, y1)
        restricts the walk to those pixel rows."""
        s = self.scene
        dimage = np.ascontiguousarray(dimage, np.float64)
        K = s.sh_k
        out = dict(screen=np.zeros((s.n, 9)), means=np.zeros((3, s.n_pad)),
                   log_scales=np.zeros((3, s.n_pad)), quats=np.zeros((4, s.n_pad)),
                   opacity_logits=np.zeros(s.n_pad), sh=np.zeros((3, K, s.n_pad)))
        y0, y1 = (0, self.cam.height) if rows is None else rows
        self.L.or_backward_rows(self.h, int(y0), int(y1), _p(dimage),
                                *[_p(out[k]) for k in ("screen", "means", "log_scales", "quats",
                                                       "opacity_logits", "sh")])
        return out

    def blend_backward_rows(self, y0, y1, dimage, screen_grad):
        """Adds the blend backward of the pixel rows [y0, y1) to screen_grad (n x 9)."""
        assert screen_grad.dtype == np.float64 and screen_grad.shape == (self.scene.n, 9)
        dimage = np.ascontiguousarray(dimage, np.float64)
        self.L.or_blend_backward_rows(self.h, int(y0), int(y1), _p(dimage), _p(screen_grad))

    def project_backward(self, screen_grad, i0, i1, out) -> dict:
        """Parameter gradients of the Gaussians [i0, i1) from their screen
        gradient, written into `out` (the dict `backward` returns)."""
        assert screen_grad.dtype == np.float64 and screen_grad.shape == (self.scene.n, 9)
        self.L.or_project_backward(self.h, _p(screen_grad), int(i0), int(i1),
                                   *[_p(out[k]) for k in ("means", "log_scales", "quats",
                                                          "opacity_logits", "sh")])
        return out

    def camera_backward(self, screen_grad):
        """dL/d(pose) = (dL/dw, dL/dt) for the pose update R <- exp([w]x) R,
        t <- t + dt, from the screen gradient (n x 9) of this view."""
        assert screen_grad.dtype == np.float64 and screen_grad.shape == (self.scene.n, 9)
        out = np.zeros(6)
        self.L.or_camera_backward(self.h, _p(np.ascontiguousarray(screen_grad)), _p(out))
        return out


def loss(image, target, lam=0.2, with_grad=True):
    """(1 - lam) L1 + lam (1 - SSIM). Returns (loss, l1, ssim, dL/dimage or None).
    float32 inputs are read as float32 (as the CUDA path receives them); float64
    inputs keep full precision."""
    f64 = np.asarray(image).dtype == np.float64
    dt = np.float64 if f64 else np.float32
    image = np.ascontiguousarray(image, dt)
    target = np.ascontiguousarray(target, dt)
    _, H, W = image.shape
    out3 = np.zeros(3)
    d = np.zeros((3, H, W)) if with_grad else None
    fn = lib().or_loss_f64 if f64 else lib().or_loss
    rc = fn(H, W, _p(image), _p(target), float(lam), _p(out3), _p(d))
    if rc != 0:
        raise ValueError("oracle rejected the loss inputs")
    return out3[0], out3[1], out3[2], d


def adam(p, g, m, v, lr, step, beta1=0.9, beta2=0.999, eps=1e-8):
    """One Adam step in float64 on copies; returns (p, g, m, v)."""
    p, g, m, v = (np.array(a, dtype=np.float64, copy=True).reshape(-1) for a in (p, g, m, v))
    lib().or_adam(p.size, _p(p), _p(g), _p(m), _p(v), lr, beta1, beta2, eps, int(step))
    return p, g, m, v


def blend_screen(screen, order, px, py, bg=(0.0, 0.0, 0.0), dldI=None):
    """Blend one pixel over explicit screen-space Gaussians (n x 9) in `order`."""
    screen = np.ascontiguousarray(screen, np.float64)
    order = np.ascontiguousarray(order, np.int32)
    bg = np.ascontiguousarray(bg, np.float64)
    rgb = np.zeros(3)
    T = np.zeros(1)
    n = screen.shape[0]
    sgrad = np.zeros((n, 9)) if dldI is not None else None
    dl = None if dldI is None else np.ascontiguousarray(dldI, np.float64)
    lib().or_blend_screen(n, _p(screen), order.size, _p(order), float(px), float(py), _p(bg),
                          _p(dl), _p(rgb), _p(T), _p(sgrad))
    return rgb, T[0], sgrad


def sh_basis(degree, dirs):
    dirs = np.ascontiguousarray(dirs, np.float64).reshape(-1, 3)
    out = np.zeros((dirs.shape[0], 16))
    lib().or_sh_basis(degree, dirs.shape[0], _p(dirs), _p(out))
    return out


def rotation_cov(q, ls):
    q = np.ascontiguousarray(q, np.float64)
    ls = np.ascontiguousarray(ls, np.float64)
    R = np.zeros(9)
    S = np.zeros(9)
    lib().or_rotation_cov(_p(q), _p(ls), _p(R), _p(S))
    return R.reshape(3, 3), S.reshape(3, 3)


def full_loss(scene, cam, target, lam=0.2):
    """Scalar training loss of `scene` seen by `cam` against `target` (render + loss)."""
    o = Oracle(scene, cam)
    r = o.render()
    L, _, _, _ = loss(r["image"], np.asarray(target, np.float64), lam, with_grad=False)
    return L


__all__ = ["Oracle", "loss", "adam", "blend_screen", "sh_basis", "rotation_cov", "camera", "lib"]


# ------------------------------------------------------------ density control
# Adaptive density control between training steps, after the study notes
# (bailiping.com) slides "Where to add capacity" / "A separate heuristic" and
# "How a computer rebuilds a real place ... Gaussian Splats" (taosengine.com),
# section "Densification": plain float64 numpy, one Gaussian at a time in
# index order.

def densify_stats(screen_grad, touched):
    """This view's contribution to the densification statistics: the norm of
    dL/dmean2d (columns 0, 1 of the n x 9 screen gradient) and a count of 1 for
    every Gaussian the view touched."""
    sg = np.asarray(screen_grad, np.float64)
    vis = np.asarray(touched) > 0
    norm = np.where(vis, np.sqrt(sg[:, 0] ** 2 + sg[:, 1] ** 2), 0.0)
    return norm, vis.astype(np.int64)


def _rotation(q):
    """Rotation matrix of the normalised quaternion (w, x, y, z)."""
    w, x, y, z = np.asarray(q, np.float64) / np.linalg.norm(q)
    return np.array([[1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)],
                     [2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)],
                     [2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)]])


def densify(params, m, v, n, grad_accum, view_count, normals, grad_threshold, scale_threshold,
            min_opacity):
    """One densification pass. params / m / v: dicts of planar arrays (groups as
    in the scene layout, last axis >= n). Returns (params, m, v, n_out) with the
    last axis exactly n_out: kept Gaussians in index order, then clones in
    parent order, then split children (child 0, child 1) in parent order.

    Per Gaussian: pruned if logit < logit(min_opacity); else, if it was seen
    and its average screen-gradient norm reaches grad_threshold, cloned when
    its largest log-scale is at most log(scale_threshold) and split otherwise:
    two children at mean + R S z_k (z_k the given N(0,1) draws), log-scales
    minus ln 1.6. Kept Gaussians keep their moments, new ones start at zero."""
    groups = ("means", "log_scales", "quats", "opacity_logits", "sh")
    logit_thr = math.log(min_opacity / (1.0 - min_opacity))
    log_scale_thr = math.log(scale_threshold)
    kept, clones, children = [], [], []
    for i in range(n):
        logit = float(params["opacity_logits"][..., i])
        if logit < logit_thr:
            continue
        cnt = int(view_count[i])
        dense = cnt > 0 and float(grad_accum[i]) / cnt >= grad_threshold
        ls = np.asarray(params["log_scales"][:, i], np.float64)
        if dense and ls.max() > log_scale_thr:
            R = _rotation(params["quats"][:, i])
            S = np.diag(np.exp(ls))
            mu = np.asarray(params["means"][:, i], np.float64)
            for k in range(2):
                z = np.asarray(normals[i, k], np.float64)
                children.append((i, mu + R @ S @ z, ls - math.log(1.6)))
            continue
        kept.append(i)
        if dense:
            clones.append(i)
    n_out = len(kept) + len(clones) + len(children)
    out_p, out_m, out_v = {}, {}, {}
    for g in groups:
        shape = params[g].shape[:-1] + (n_out,)
        out_p[g] = np.zeros(shape)
        out_m[g] = np.zeros(shape)
        out_v[g] = np.zeros(shape)
        col = 0
        for i in kept:
            out_p[g][..., col] = params[g][..., i]
            out_m[g][..., col] = m[g][..., i]
            out_v[g][..., col] = v[g][..., i]
            col += 1
        for i in clones:
            out_p[g][..., col] = params[g][..., i]
            col += 1
        for (i, mean, ls) in children:
            if g == "means":
                out_p[g][..., col] = mean
            elif g == "log_scales":
                out_p[g][..., col] = ls
            else:
                out_p[g][..., col] = params[g][..., i]
            col += 1
    return out_p, out_m, out_v, n_out


def relocate(params, m, v, n, normals, dead_opacity=0.02, donor_opacity=0.4, max_pairs=None):
    """Recycling the dead ("How a computer rebuilds a real place ... Gaussian
    Splats", section "Densification: cloning the busy blobs, recycling the
    dead"), with the count fixed. Dead: opacity below dead_opacity; donors:
    opacity above donor_opacity (both decided on the logit in float64). The
    donors are taken largest first (largest log-scale, ties by index), the dead
    in index order, and the j-th dead is paired with the j-th donor, for
    j < min(dead, donors, max_pairs, len(normals)). For a pair (d, b): slot d
    becomes a copy of b placed at mean_b + R_b S_b z_j (z_j = normals[j], the
    donor's own Gaussian, as a split child is placed), both d and b take
    log-scales log_scale_b - ln 1.6 ("both halves shrink"), and both restart
    their Adam moments at zero. Every other slot is unchanged. Returns
    (params, m, v, pairs) as float64 copies (pairs: list of (d, b))."""
    groups = ("means", "log_scales", "quats", "opacity_logits", "sh")
    P = {g: np.array(params[g], np.float64, copy=True) for g in groups}
    M = {g: np.array(m[g], np.float64, copy=True) for g in groups}
    V = {g: np.array(v[g], np.float64, copy=True) for g in groups}
    dead_thr = math.log(dead_opacity / (1.0 - dead_opacity))
    donor_thr = math.log(donor_opacity / (1.0 - donor_opacity))
    logits = P["opacity_logits"][..., :n]
    dead = [i for i in range(n) if logits[i] < dead_thr]
    donors = [i for i in range(n) if logits[i] > donor_thr]
    size = {i: float(np.max(np.float32(P["log_scales"][:, i]))) for i in donors}
    donors.sort(key=lambda i: (-size[i], i))
    count = min(len(dead), len(donors), len(normals))
    if max_pairs is not None:
        count = min(count, max_pairs)
    pairs = []
    for j in range(count):
        d, b = dead[j], donors[j]
        ls_b = P["log_scales"][:, b].copy()
        R = _rotation(P["quats"][:, b])
        child = P["means"][:, b] + R @ np.diag(np.exp(ls_b)) @ np.asarray(normals[j], np.float64)
        for g in groups:
            P[g][..., d] = P[g][..., b]
        P["means"][:, d] = child
        P["log_scales"][:, d] = ls_b - math.log(1.6)
        P["log_scales"][:, b] = ls_b - math.log(1.6)
        for g in groups:
            for slot in (d, b):
                M[g][..., slot] = 0.0
                V[g][..., slot] = 0.0
        pairs.append((d, b))
    return P, M, V, pairs


def opacity_reset(logits, m, v, max_opacity):
    """logit = min(logit, logit(max_opacity)); the moments of the logits set to zero."""
    cap = math.log(max_opacity / (1.0 - max_opacity))
    logits = np.minimum(np.asarray(logits, np.float64), cap)
    return logits, np.zeros_like(np.asarray(m, np.float64)), np.zeros_like(np.asarray(v, np.float64))


# --------------------------------------------------- Charbonnier + exposure
def charbonnier_loss(image, target, gain, bias, delta=0.03):
    """Robust photometric loss with a per-photo exposure correction, after "How a
    computer rebuilds a real place ... Gaussian Splats" (taosengine.com), the
    loss paragraph before "The chain rule, in one breath": per pixel p and
    channel c, err = gain_c C + bias_c - target, root = sqrt(err^2 + delta^2),
    pixel loss = sum_c root - 3 delta; the image loss is the mean over the H W
    pixels. Returns (loss, dL/dimage [3,H,W], dL/dgain [3], dL/dbias [3]) in
    float64."""
    x = np.asarray(image, np.float64)
    y = np.asarray(target, np.float64)
    g = np.asarray(gain, np.float64).reshape(3, 1, 1)
    b = np.asarray(bias, np.float64).reshape(3, 1, 1)
    P = x.shape[1] * x.shape[2]
    err = g * x + b - y
    root = np.sqrt(err * err + delta * delta)
    loss = float((root.sum(axis=0) - 3.0 * delta).sum() / P)
    slope = err / root
    d_image = g * slope / P
    d_gain = (slope * x).sum(axis=(1, 2)) / P
    d_bias = slope.sum(axis=(1, 2)) / P
    return loss, d_image, d_gain, d_bias
