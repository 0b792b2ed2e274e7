"""ctypes binding of the C ABI in include/gs_api.h.

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the `stream` argument, and a non-OK status becomes an
exception carrying gs_last_error(). Every step of the path runs in the CUDA
library; there is no fallback of any kind, so a missing or unloadable library
raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgsb200.so")

GS_OK, GS_ERR_INVALID_ARG, GS_ERR_CAPACITY, GS_ERR_CUDA, GS_ERR_DEVICE = range(5)
_STATUS = {0: "GS_OK", 1: "GS_ERR_INVALID_ARG", 2: "GS_ERR_CAPACITY", 3: "GS_ERR_CUDA",
           4: "GS_ERR_DEVICE"}

EXPORTED = ("gs_create", "gs_destroy", "gs_last_error", "gs_preprocess", "gs_render_forward",
            "gs_loss_l1_dssim", "gs_render_backward", "gs_render_backward_adam", "gs_adam_step",
            "gs_profile_enable",
            "gs_profile_read", "gs_stage_name", "gs_debug_preprocess", "gs_debug_sorted",
            "gs_debug_screen_grads", "gs_set_option", "gs_loss_l1_dssim_noalloc",
            "gs_set_densify_stats", "gs_densify", "gs_opacity_reset", "gs_loss_charbonnier",
            "gs_adam_step_reduce", "gs_shared_alloc", "gs_shared_open", "gs_shared_close",
            "gs_shared_free", "gs_set_camera_grad", "gs_relocate", "gs_render_backward_screen",
            "gs_get_view", "gs_shared_handle", "gs_adam_step_views")
GS_SHARED_HANDLE_BYTES = 64
MAX_RANKS = 8
GS_OPTION_OPACITY_RECT = 1
GS_OPTION_DETERMINISTIC = 2
GS_OPTION_MIP_COMPENSATION = 3
PROFILE_TIME = 1   # GS_PROFILE_TIME
PROFILE_COUNT = 2  # GS_PROFILE_COUNT
STAGES = ("preprocess", "scan", "duplicate", "sort", "ranges", "blend_forward", "loss",
          "blend_backward", "preprocess_backward", "backward_adam", "depth_sort", "camera_backward",
          "views_adam")
GROUPS = ("means", "log_scales", "quats", "opacity_logits", "sh")


class GsError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class GsCamera(ctypes.Structure):
    _fields_ = [("width", ctypes.c_int32), ("height", ctypes.c_int32),
                ("fx", ctypes.c_float), ("fy", ctypes.c_float),
                ("cx", ctypes.c_float), ("cy", ctypes.c_float),
                ("R", ctypes.c_float * 9), ("t", ctypes.c_float * 3),
                ("campos", ctypes.c_float * 3), ("bg", ctypes.c_float * 3),
                ("near_z", ctypes.c_float)]


class GsParams(ctypes.Structure):
    _fields_ = [("means", ctypes.c_void_p), ("log_scales", ctypes.c_void_p),
                ("quats", ctypes.c_void_p), ("opacity_logits", ctypes.c_void_p),
                ("sh", ctypes.c_void_p), ("n", ctypes.c_int64), ("n_pad", ctypes.c_int64),
                ("sh_degree", ctypes.c_int32), ("active_degree", ctypes.c_int32)]


class GsGrads(ctypes.Structure):
    _fields_ = [("means", ctypes.c_void_p), ("log_scales", ctypes.c_void_p),
                ("quats", ctypes.c_void_p), ("opacity_logits", ctypes.c_void_p),
                ("sh", ctypes.c_void_p)]


class GsView(ctypes.Structure):
    """One rank's view (gs_view): device addresses of its screen records, raw
    screen sums, touched counts, clamp flags and camera record."""
    _fields_ = [("screen", ctypes.c_void_p), ("sums", ctypes.c_void_p), ("touched", ctypes.c_void_p),
                ("clamped", ctypes.c_void_p), ("camera", ctypes.c_void_p)]
    FIELDS = ("screen", "sums", "touched", "clamped", "camera")


_lib = None


def load(path: str = LIB_PATH):
    """Loads the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing (run __graft_entry__.build())")
    L = ctypes.CDLL(path)
    P, I32, I64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    L.gs_create.argtypes = [ctypes.POINTER(P), I64, I64, I32, I32]
    L.gs_destroy.argtypes = [P]
    L.gs_destroy.restype = None
    L.gs_last_error.argtypes = [P]
    L.gs_last_error.restype = ctypes.c_char_p
    L.gs_preprocess.argtypes = [P, ctypes.POINTER(GsParams), ctypes.POINTER(GsCamera), P]
    L.gs_render_forward.argtypes = [P, ctypes.POINTER(GsCamera), P, P, P, ctypes.POINTER(I64), P]
    L.gs_loss_l1_dssim.argtypes = [P, P, P, I32, I32, F, P, P, P]
    L.gs_render_backward.argtypes = [P, ctypes.POINTER(GsParams), ctypes.POINTER(GsCamera), P, P, P,
                                     ctypes.POINTER(GsGrads), P]
    L.gs_render_backward_adam.argtypes = [P, ctypes.POINTER(GsParams), ctypes.POINTER(GsCamera), P, P, P,
                                          ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads),
                                          ctypes.POINTER(GsGrads), ctypes.POINTER(F), F, F, F, I32, P]
    L.gs_adam_step.argtypes = [P, P, P, P, I64, F, F, F, F, I32, P]
    L.gs_set_densify_stats.argtypes = [P, P, P]
    L.gs_densify.argtypes = [P, ctypes.POINTER(GsParams), ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads),
                             P, P, P, F, F, F, ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads),
                             ctypes.POINTER(GsGrads), I64, ctypes.POINTER(I64), P]
    L.gs_opacity_reset.argtypes = [P, P, P, I64, F, P]
    L.gs_loss_charbonnier.argtypes = [P, P, P, I32, I32, ctypes.POINTER(F), ctypes.POINTER(F), F, P, P, P]
    PP = ctypes.POINTER(P)
    L.gs_adam_step_reduce.argtypes = [P, P, P, I64, PP, I32, PP, I32, I32, F, F, F, F, F, I32, P]
    L.gs_shared_alloc.argtypes = [I64, PP, ctypes.c_char_p]
    L.gs_shared_open.argtypes = [ctypes.c_char_p, PP]
    L.gs_shared_close.argtypes = [P]
    L.gs_shared_free.argtypes = [P]
    L.gs_set_camera_grad.argtypes = [P, P]
    L.gs_relocate.argtypes = [P, ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads),
                              I64, I64, I32, P, I64, F, F, ctypes.POINTER(I64), P]
    L.gs_render_backward_screen.argtypes = [P, ctypes.POINTER(GsParams), ctypes.POINTER(GsCamera), P, P, P, P]
    L.gs_get_view.argtypes = [P, ctypes.POINTER(GsView)]
    L.gs_shared_handle.argtypes = [P, ctypes.c_char_p]
    L.gs_adam_step_views.argtypes = [P, ctypes.POINTER(GsParams), ctypes.POINTER(GsView), I32, I64, I64,
                                     ctypes.POINTER(GsGrads), I32, ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads),
                                     ctypes.POINTER(F), F, F, F, F, I32, P]
    L.gs_set_option.argtypes = [P, I32, I32]
    L.gs_set_option.restype = ctypes.c_int
    L.gs_loss_l1_dssim_noalloc.argtypes = [P, P, I32, I32, F, P, P, P]
    L.gs_loss_l1_dssim_noalloc.restype = ctypes.c_int
    L.gs_profile_enable.argtypes = [P, I32]
    L.gs_profile_read.argtypes = [P, P, P, P, P]
    L.gs_stage_name.argtypes = [I32]
    L.gs_stage_name.restype = ctypes.c_char_p
    L.gs_debug_preprocess.argtypes = [P] * 10
    L.gs_debug_sorted.argtypes = [P] * 5
    L.gs_debug_screen_grads.argtypes = [P] * 3
    for name in EXPORTED:
        if name not in ("gs_destroy", "gs_last_error", "gs_stage_name"):
            getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def camera_struct(cam) -> GsCamera:
    c = GsCamera()
    c.width, c.height = int(cam.width), int(cam.height)
    c.fx, c.fy, c.cx, c.cy = float(cam.fx), float(cam.fy), float(cam.cx), float(cam.cy)
    for i, v in enumerate(np.asarray(cam.R, np.float32).reshape(-1)):
        c.R[i] = float(v)
    for name in ("t", "campos", "bg"):
        arr = getattr(c, name)
        for i, v in enumerate(np.asarray(getattr(cam, name), np.float32).reshape(-1)):
            arr[i] = float(v)
    c.near_z = float(cam.near_z)
    return c


class Context:
    """Owns one gs_ctx; methods mirror the C entry points one to one."""

    def __init__(self, max_gaussians, max_entries, max_width, max_height):
        self.L = load()
        h = ctypes.c_void_p()
        st = self.L.gs_create(ctypes.byref(h), int(max_gaussians), int(max_entries), int(max_width),
                              int(max_height))
        if st != GS_OK:
            raise GsError(st, "gs_create failed")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            self.L.gs_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, st):
        if st != GS_OK:
            raise GsError(st, self.L.gs_last_error(self.h).decode())

    def set_option(self, option, value):
        self._check(self.L.gs_set_option(self.h, int(option), int(value)))

    def loss_charbonnier(self, image, target, gain, bias, out, dloss_dimage=None, delta=0.03, stream=None):
        _, H, W = image.shape
        g = (ctypes.c_float * 3)(*[float(x) for x in gain])
        b = (ctypes.c_float * 3)(*[float(x) for x in bias])
        self._check(self.L.gs_loss_charbonnier(self.h, _ptr(image), _ptr(target), H, W, g, b, float(delta),
                                               _ptr(out), _ptr(dloss_dimage), _stream(stream)))

    def render_backward_screen(self, params: GsParams, cam: GsCamera, final_T, n_contrib, dloss_dimage,
                               stream=None):
        """The blend backward alone; the raw screen sums stay in the context as its view."""
        self._check(self.L.gs_render_backward_screen(self.h, ctypes.byref(params), ctypes.byref(cam),
                                                     _ptr(final_T), _ptr(n_contrib), _ptr(dloss_dimage),
                                                     _stream(stream)))

    def view(self) -> GsView:
        """This context's view buffers (device addresses)."""
        v = GsView()
        self._check(self.L.gs_get_view(self.h, ctypes.byref(v)))
        return v

    def adam_step_views(self, params: GsParams, views, g_lo, g_hi, copies, exp_avg: GsGrads, exp_avg_sq: GsGrads,
                        lrs, step, grad_scale=None, beta1=0.9, beta2=0.999, eps=1e-8, stream=None):
        """gs_adam_step_views: views = [GsView] in rank order, copies = [GsGrads] of the
        other ranks' parameter groups; grad_scale defaults to 1 / len(views)."""
        if not 1 <= len(views) <= MAX_RANKS or len(copies) > MAX_RANKS:
            raise ValueError(f"1..{MAX_RANKS} views and at most {MAX_RANKS} copies")
        va = (GsView * len(views))(*views)
        ca = (GsGrads * max(1, len(copies)))(*copies) if copies else None
        lr = (ctypes.c_float * 5)(*[float(x) for x in lrs])
        scale = 1.0 / len(views) if grad_scale is None else float(grad_scale)
        self._check(self.L.gs_adam_step_views(self.h, ctypes.byref(params), va, len(views), int(g_lo), int(g_hi),
                                              ca, len(copies), ctypes.byref(exp_avg), ctypes.byref(exp_avg_sq),
                                              lr, scale, float(beta1), float(beta2), float(eps), int(step),
                                              _stream(stream)))

    def set_camera_grad(self, out):
        """Every later backward writes this view's pose gradient (dL/dw, dL/dt) to
        `out` (6 float64 on the device); None turns it off."""
        self._out_cam = out  # kept alive while the context points at it
        self._check(self.L.gs_set_camera_grad(self.h, _ptr(out)))

    def relocate(self, params: GsGrads, m: GsGrads, v: GsGrads, n, n_pad, sh_degree, normals, max_pairs,
                 dead_opacity=0.02, donor_opacity=0.4, stream=None) -> int:
        """gs_relocate in place; returns the number of pairs made."""
        n_pairs = ctypes.c_int64(0)
        self._check(self.L.gs_relocate(self.h, ctypes.byref(params), ctypes.byref(m), ctypes.byref(v), int(n),
                                       int(n_pad), int(sh_degree), _ptr(normals), int(max_pairs),
                                       float(dead_opacity), float(donor_opacity), ctypes.byref(n_pairs),
                                       _stream(stream)))
        return n_pairs.value

    def set_densify_stats(self, grad_accum, view_count):
        self._check(self.L.gs_set_densify_stats(self.h, _ptr(grad_accum), _ptr(view_count)))

    def densify(self, params: GsParams, m_in: GsGrads, v_in: GsGrads, grad_accum, view_count, normals,
                grad_threshold, scale_threshold, min_opacity, out: GsGrads, m_out: GsGrads, v_out: GsGrads,
                out_n_pad, stream=None) -> int:
        n_out = ctypes.c_int64(0)
        self._check(self.L.gs_densify(self.h, ctypes.byref(params), ctypes.byref(m_in), ctypes.byref(v_in),
                                      _ptr(grad_accum), _ptr(view_count), _ptr(normals),
                                      float(grad_threshold), float(scale_threshold), float(min_opacity),
                                      ctypes.byref(out), ctypes.byref(m_out), ctypes.byref(v_out),
                                      int(out_n_pad), ctypes.byref(n_out), _stream(stream)))
        return n_out.value

    def preprocess(self, params: GsParams, cam: GsCamera, stream=None):
        self._check(self.L.gs_preprocess(self.h, ctypes.byref(params), ctypes.byref(cam), _stream(stream)))

    def render_forward(self, cam: GsCamera, image, final_T, n_contrib, stream=None) -> int:
        k = ctypes.c_int64(0)
        self._check(self.L.gs_render_forward(self.h, ctypes.byref(cam), _ptr(image), _ptr(final_T),
                                             _ptr(n_contrib), ctypes.byref(k), _stream(stream)))
        return k.value

    def loss_l1_dssim(self, image, target, lam, loss_out, dloss_dimage=None, stream=None):
        _, H, W = image.shape
        self._check(self.L.gs_loss_l1_dssim(self.h, _ptr(image), _ptr(target), H, W, float(lam),
                                            _ptr(loss_out), _ptr(dloss_dimage), _stream(stream)))

    def render_backward(self, params: GsParams, cam: GsCamera, final_T, n_contrib, dloss_dimage,
                        grads: GsGrads, stream=None):
        self._check(self.L.gs_render_backward(self.h, ctypes.byref(params), ctypes.byref(cam),
                                              _ptr(final_T), _ptr(n_contrib), _ptr(dloss_dimage),
                                              ctypes.byref(grads), _stream(stream)))

    def render_backward_adam(self, params: GsParams, cam: GsCamera, final_T, n_contrib, dloss_dimage,
                             grads, exp_avg: GsGrads, exp_avg_sq: GsGrads, lrs, step,
                             beta1=0.9, beta2=0.999, eps=1e-8, stream=None):
        """grads: a GsGrads with an accumulated gradient (zeroed by the call), or
        None when there is none (no gradient buffer is read or written)."""
        lr = (ctypes.c_float * 5)(*[float(x) for x in lrs])
        g = None if grads is None else ctypes.byref(grads)
        self._check(self.L.gs_render_backward_adam(
            self.h, ctypes.byref(params), ctypes.byref(cam), _ptr(final_T), _ptr(n_contrib),
            _ptr(dloss_dimage), g, ctypes.byref(exp_avg), ctypes.byref(exp_avg_sq),
            lr, float(beta1), float(beta2), float(eps), int(step), _stream(stream)))

    def profile_enable(self, on=True, count_pairs=False):
        """Stage timing of the production kernels (on); count_pairs also makes
        the two blends count their (pixel, Gaussian) pairs, through counting
        variants whose times then replace the production kernels'."""
        self._check(self.L.gs_profile_enable(self.h, (PROFILE_TIME if on else 0) |
                                             (PROFILE_COUNT if count_pairs else 0)))

    def profile_read(self) -> dict:
        n = len(STAGES)
        ms = (ctypes.c_double * n)()
        launches = (ctypes.c_int64 * n)()
        work = (ctypes.c_int64 * n)()
        blended = (ctypes.c_int64 * n)()
        self._check(self.L.gs_profile_read(self.h, ms, launches, work, blended))
        return {STAGES[k]: {"ms": ms[k], "launches": launches[k], "work": work[k], "blended": blended[k]}
                for k in range(n)}

    def debug_preprocess(self, mean2d=None, conic=None, opacity=None, rgb=None, depth=None, rect=None,
                         touched=None, clamped=None, stream=None):
        self._check(self.L.gs_debug_preprocess(self.h, _ptr(mean2d), _ptr(conic), _ptr(opacity),
                                               _ptr(rgb), _ptr(depth), _ptr(rect), _ptr(touched),
                                               _ptr(clamped), _stream(stream)))

    def debug_sorted(self, ids=None, tiles=None, ranges=None, stream=None):
        self._check(self.L.gs_debug_sorted(self.h, _ptr(ids), _ptr(tiles), _ptr(ranges), _stream(stream)))

    def debug_screen_grads(self, out, stream=None):
        self._check(self.L.gs_debug_screen_grads(self.h, _ptr(out), _stream(stream)))


def adam_step(param, grad, m, v, lr, step, beta1=0.9, beta2=0.999, eps=1e-8, stream=None):
    L = load()
    st = L.gs_adam_step(_ptr(param), _ptr(grad), _ptr(m), _ptr(v), param.numel(), float(lr),
                        float(beta1), float(beta2), float(eps), int(step), _stream(stream))
    if st != GS_OK:
        raise GsError(st, "gs_adam_step rejected its arguments")


def adam_step_reduce(param, m, v, grads, copies, lr, step, grad_scale=None, zero_grads=False, beta1=0.9,
                     beta2=0.999, eps=1e-8, stream=None):
    """gs_adam_step_reduce over the tensors param, m, v (this rank's piece of its
    shard). grads / copies: device addresses (ints) of the same piece in every
    rank's gradient buffer and in the other ranks' parameter buffers. grad_scale
    defaults to 1 / len(grads)."""
    L = load()
    if not 1 <= len(grads) <= MAX_RANKS or len(copies) > MAX_RANKS:
        raise ValueError(f"1..{MAX_RANKS} gradient sources and at most {MAX_RANKS} copies")
    scale = 1.0 / len(grads) if grad_scale is None else float(grad_scale)
    g = (ctypes.c_void_p * max(1, len(grads)))(*[ctypes.c_void_p(int(x)) for x in grads])
    c = (ctypes.c_void_p * max(1, len(copies)))(*[ctypes.c_void_p(int(x)) for x in copies])
    st = L.gs_adam_step_reduce(_ptr(param), _ptr(m), _ptr(v), param.numel(), g, len(grads), c, len(copies),
                               int(bool(zero_grads)), scale, float(lr), float(beta1), float(beta2), float(eps),
                               int(step), _stream(stream))
    if st != GS_OK:
        raise GsError(st, "gs_adam_step_reduce rejected its arguments")


class SharedBuffer:
    """float32 device memory that other processes can map (gs_shared_alloc), freed
    with the object. `.tensor` is a torch view of it; `.handle` the bytes to send
    to the other ranks; `.ptr` its device address."""

    def __init__(self, numel):
        L = load()
        self.numel = int(numel)
        p = ctypes.c_void_p()
        h = ctypes.create_string_buffer(GS_SHARED_HANDLE_BYTES)
        st = L.gs_shared_alloc(4 * self.numel, ctypes.byref(p), h)
        if st != GS_OK:
            raise GsError(st, "gs_shared_alloc failed")
        self.ptr = int(p.value)
        self.handle = bytes(h.raw)
        import torch
        self.tensor = torch.as_tensor(self, device=f"cuda:{torch.cuda.current_device()}")

    @property
    def __cuda_array_interface__(self):
        return {"shape": (self.numel,), "typestr": "<f4", "data": (self.ptr, False), "version": 3,
                "strides": None}

    def __del__(self):
        if getattr(self, "ptr", 0) and _lib is not None:
            _lib.gs_shared_free(ctypes.c_void_p(self.ptr))
            self.ptr = 0


def shared_open(handle: bytes) -> int:
    """Maps another process's SharedBuffer from its handle; returns the device address."""
    L = load()
    if len(handle) != GS_SHARED_HANDLE_BYTES:
        raise ValueError("bad handle size")
    p = ctypes.c_void_p()
    st = L.gs_shared_open(handle, ctypes.byref(p))
    if st != GS_OK:
        raise GsError(st, "gs_shared_open failed")
    return int(p.value)


def shared_handle(ptr: int) -> bytes:
    """The IPC handle of the device allocation starting at ptr (for shared_open on
    another rank)."""
    h = ctypes.create_string_buffer(GS_SHARED_HANDLE_BYTES)
    st = load().gs_shared_handle(ctypes.c_void_p(int(ptr)), h)
    if st != GS_OK:
        raise GsError(st, "gs_shared_handle failed")
    return bytes(h.raw)


def shared_close(ptr: int):
    st = load().gs_shared_close(ctypes.c_void_p(int(ptr)))
    if st != GS_OK:
        raise GsError(st, "gs_shared_close failed")


def opacity_reset(logits, m, v, max_opacity=0.01, stream=None):
    L = load()
    st = L.gs_opacity_reset(_ptr(logits), _ptr(m), _ptr(v), logits.numel(), float(max_opacity),
                            _stream(stream))
    if st != GS_OK:
        raise GsError(st, "gs_opacity_reset rejected its arguments")
