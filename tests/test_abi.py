"""The C ABI library loads on a machine without a GPU and exports every entry
point the public header declares; argument checks that come before any CUDA
call are exercised here too (no compute call is made)."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gs_api.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gs_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_five_steps():
    names = declared_functions()
    for n in ("gs_preprocess", "gs_render_forward", "gs_loss_l1_dssim", "gs_render_backward",
              "gs_adam_step", "gs_create", "gs_destroy", "gs_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    lib = ctypes.CDLL(native.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(native.EXPORTED) <= set(declared_functions())


def test_create_rejects_bad_sizes_without_touching_the_device():
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    lib = native.load()
    h = ctypes.c_void_p()
    for args in ((0, 10, 16, 16), (10, 0, 16, 16), (10, 10, 0, 16), (10, 1 << 30, 16, 16)):
        assert lib.gs_create(ctypes.byref(h), *args) == native.GS_ERR_INVALID_ARG
        assert h.value is None
    assert lib.gs_adam_step(None, None, None, None, -1, 1e-3, 0.9, 0.999, 1e-8, 1, None) == \
        native.GS_ERR_INVALID_ARG
    assert lib.gs_adam_step(None, None, None, None, 0, 1e-3, 0.9, 0.999, 1e-8, 0, None) == \
        native.GS_ERR_INVALID_ARG


def test_stage_names_match_the_binding():
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    L = native.load()
    assert [L.gs_stage_name(k).decode() for k in range(len(native.STAGES))] == list(native.STAGES)
    assert L.gs_stage_name(len(native.STAGES)).decode() == ""


def test_header_constants_match_the_binding():
    """The option and profiling flag values the binding passes are the header's."""
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    text = open(HEADER).read()
    defines = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(GS_[A-Z_]+) = (\d+)", text)}
    assert defines["GS_PROFILE_TIME"] == native.PROFILE_TIME
    assert defines["GS_PROFILE_COUNT"] == native.PROFILE_COUNT
    for name in ("GS_OPTION_OPACITY_RECT", "GS_OPTION_DETERMINISTIC", "GS_OPTION_MIP_COMPENSATION"):
        assert defines[name] == getattr(native, name), name
    L = native.load()
    assert L.gs_profile_enable(None, native.PROFILE_TIME) == native.GS_ERR_INVALID_ARG


def test_new_entry_points_check_their_arguments_on_the_host():
    """The data-parallel, shared-memory, camera-gradient and recycling entry
    points reject bad arguments before any CUDA call (so this runs without a GPU)."""
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    L = native.load()
    bad = native.GS_ERR_INVALID_ARG
    P = ctypes.c_void_p
    grads = (P * 1)(P(16))
    # gs_adam_step_reduce: no gradient source, too many, negative count, step 0, bad betas
    for n_grads, count, step, b1 in ((0, 4, 1, 0.9), (9, 4, 1, 0.9), (1, -1, 1, 0.9), (1, 4, 0, 0.9),
                                     (1, 4, 1, 1.0)):
        assert L.gs_adam_step_reduce(None, None, None, count, grads, n_grads, None, 0, 0, 1.0, 1e-3, b1,
                                     0.999, 1e-8, step, None) == bad
    # copies requested with no array
    assert L.gs_adam_step_reduce(None, None, None, 4, grads, 1, None, 1, 0, 1.0, 1e-3, 0.9, 0.999, 1e-8, 1,
                                 None) == bad
    # shared buffers: no size, no outputs, no handle, nothing to close or free
    p = P()
    h = ctypes.create_string_buffer(native.GS_SHARED_HANDLE_BYTES)
    assert L.gs_shared_alloc(0, ctypes.byref(p), h) == bad
    assert L.gs_shared_alloc(64, None, h) == bad
    assert L.gs_shared_open(None, ctypes.byref(p)) == bad
    assert L.gs_shared_close(None) == bad
    assert L.gs_shared_free(None) == bad
    # camera gradient and recycling need a context
    assert L.gs_set_camera_grad(None, None) == bad
    n_pairs = ctypes.c_int64(-1)
    g = native.GsGrads()
    assert L.gs_relocate(None, ctypes.byref(g), ctypes.byref(g), ctypes.byref(g), 0, 0, 0, None, 0, 0.02, 0.4,
                         ctypes.byref(n_pairs), None) == bad
