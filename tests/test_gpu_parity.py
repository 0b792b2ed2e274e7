"""CUDA path against the float64 oracle on the same seeded inputs, through the C ABI.

Tolerances: sort order and ranges bit-exact; rendered pixels within 1e-4
absolute (pixels whose oracle walk came within a hair of a threshold are
excluded and counted); loss within 1e-5 relative; per-group gradients within
1e-3 relative L2; Adam within float32 rounding of the float64 update.
"""
import numpy as np
import pytest

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

PIX_TOL = 1e-4
LOSS_RTOL = 1e-5
GRAD_RL2 = 1e-3


@pytest.fixture(scope="module")
def gs():
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import native, model
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    native.load()
    return native, model


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    return t.detach().cpu().numpy()


class DeviceRun:
    """Preprocess + forward of one scene/camera through the C ABI."""

    def __init__(self, native, model, scene, cam, max_entries=None, active_degree=None, opacity_rect=False,
                 mip_comp=False):
        self.native = native
        self.m = model.GaussianModel(scene, active_degree=active_degree)
        self.cam = cam
        self.cs = native.camera_struct(cam)
        o = oracle.Oracle(scene, cam, active_degree, opacity_rect=opacity_rect, mip_comp=mip_comp)
        self.oracle = o
        K_or = oracle.lib().or_num_entries(o.h)
        self.ctx = native.Context(scene.n_pad, max_entries or max(16, 2 * K_or + 16), cam.width, cam.height)
        if opacity_rect:
            self.ctx.set_option(native.GS_OPTION_OPACITY_RECT, 1)
        if mip_comp:
            self.ctx.set_option(native.GS_OPTION_MIP_COMPENSATION, 1)
        H, W = cam.height, cam.width
        self.image = torch.empty((3, H, W), device="cuda")
        self.T = torch.empty((H, W), device="cuda")
        self.nc = torch.empty((H, W), dtype=torch.int32, device="cuda")
        self.ctx.preprocess(self.m.params_struct(), self.cs)
        self.K = self.ctx.render_forward(self.cs, self.image, self.T, self.nc)
        torch.cuda.synchronize()

    def preprocess_out(self):
        n = self.m.n
        out = dict(mean2d=torch.empty((n, 2), device="cuda"), conic=torch.empty((n, 3), device="cuda"),
                   opacity=torch.empty(n, device="cuda"), rgb=torch.empty((n, 3), device="cuda"),
                   depth=torch.empty(n, device="cuda"),
                   rect=torch.empty((n, 4), dtype=torch.int32, device="cuda"),
                   touched=torch.empty(n, dtype=torch.int32, device="cuda"),
                   clamped=torch.empty(n, dtype=torch.uint8, device="cuda"))
        self.ctx.debug_preprocess(**out)
        torch.cuda.synchronize()
        return {k: host(v) for k, v in out.items()}

    def sorted_out(self):
        tx, ty = (self.cam.width + 15) // 16, (self.cam.height + 15) // 16
        ids = torch.empty(max(self.K, 1), dtype=torch.int32, device="cuda")
        tiles = torch.empty(max(self.K, 1), dtype=torch.int32, device="cuda")
        ranges = torch.empty((tx * ty, 2), dtype=torch.int32, device="cuda")
        self.ctx.debug_sorted(ids, tiles, ranges)
        torch.cuda.synchronize()
        return host(ids)[: self.K], host(tiles)[: self.K], host(ranges)

    def backward(self, dimage):
        d = dev(dimage)
        self.m.grad_flat.zero_()
        self.ctx.render_backward(self.m.params_struct(), self.cs, self.T, self.nc, d, self.m.grads_struct())
        sg = torch.empty((self.m.n, 9), device="cuda")
        self.ctx.debug_screen_grads(sg)
        torch.cuda.synchronize()
        return {k: host(v) for k, v in self.m.grads.items()}, host(sg)


def rel_l2(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


SCENES = {"tiny": lambda: (scenes.tiny(), 0), "small": lambda: (scenes.small(), 0)}


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_preprocess_matches_oracle(gs, name):
    native, model = gs
    s, ci = SCENES[name]()
    run = DeviceRun(native, model, s, s.cameras[ci])
    g = run.preprocess_out()
    o = run.oracle.preprocess()
    np.testing.assert_array_equal(g["touched"], o["touched"])
    vis = o["touched"] > 0
    np.testing.assert_array_equal(g["rect"][vis], o["rect"][vis])
    np.testing.assert_array_equal(g["depth"].view(np.uint32), o["depth_key"].view(np.uint32))
    np.testing.assert_allclose(g["mean2d"][vis], o["screen"][vis, 0:2], rtol=0, atol=1e-4)
    np.testing.assert_allclose(g["conic"][vis], o["screen"][vis, 2:5], rtol=1e-5,
                               atol=1e-6 * np.abs(o["screen"][vis, 2:5]).max())
    np.testing.assert_allclose(g["opacity"][vis], o["screen"][vis, 5], rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(g["rgb"][vis], o["screen"][vis, 6:9], rtol=0, atol=1e-5)
    # colour clamps agree except where the unclamped colour is within rounding of 0
    mism = (g["clamped"][vis][:, None] >> np.arange(3) & 1) != o["clamped"][vis]
    assert mism.sum() <= max(1, vis.sum() // 1000)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_sort_and_ranges_bit_exact(gs, name):
    native, model = gs
    s, ci = SCENES[name]()
    run = DeviceRun(native, model, s, s.cameras[ci])
    ids, tiles, ranges = run.sorted_out()
    o = run.oracle.sorted()
    assert run.K == o["ids"].size
    np.testing.assert_array_equal(ids, o["ids"])
    np.testing.assert_array_equal(tiles, o["tiles"])
    np.testing.assert_array_equal(ranges.astype(np.int64), o["ranges"])


def check_pixels(run, o_render):
    img, T, nc = host(run.image), host(run.T), host(run.nc)
    amb = o_render["ambiguous"].astype(bool)
    ok = ~amb
    assert amb.mean() < 0.01, f"{amb.sum()} ambiguous pixels"
    err = np.abs(img - o_render["image"])[:, ok]
    assert err.max() <= PIX_TOL, err.max()
    # T enters the pixel as T * background: compared at the pixel tolerance
    np.testing.assert_allclose(T[ok], o_render["final_T"][ok], rtol=0, atol=PIX_TOL)
    np.testing.assert_array_equal(nc[ok], o_render["n_contrib"][ok])
    # an ambiguous pixel (a decision within float32 reach of its threshold) must
    # equal the oracle's walk with some of those decisions taken the other way
    py, px = np.nonzero(amb)
    if px.size:
        n_amb = run.oracle.replay_pixels(px, py, 0)["n_amb"]
        assert n_amb.max() <= 8, n_amb.max()
        matched = np.zeros(px.size, bool)
        for mask in range(1 << int(n_amb.max())):
            rep = run.oracle.replay_pixels(px, py, mask)
            matched |= ((np.abs(img[:, py, px].T - rep["rgb"]).max(axis=1) <= PIX_TOL) &
                        (np.abs(T[py, px] - rep["T"]) <= PIX_TOL) & (nc[py, px] == rep["n_contrib"]))
        assert matched.all(), np.nonzero(~matched)[0][:10]
    return amb.sum()


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_forward_pixels_match_oracle(gs, name):
    native, model = gs
    s, ci = SCENES[name]()
    run = DeviceRun(native, model, s, s.cameras[ci])
    check_pixels(run, run.oracle.render())


def test_forward_ragged_image_and_background(gs):
    """An image size that is not a multiple of the 16-pixel tile, a coloured
    background and SH degree 3 with only degree 1 active."""
    native, model = gs
    s = scenes.small(seed=3)
    cam = scenes.look_at((0.4, 0.3, -3.2), (0.0, 0.0, 0.0), 150, 93, 140.0, bg=(0.2, 0.5, 0.9))
    run = DeviceRun(native, model, s, cam, active_degree=1)
    check_pixels(run, run.oracle.render())
    ids, _, ranges = run.sorted_out()
    o = run.oracle.sorted()
    np.testing.assert_array_equal(ids, o["ids"])
    np.testing.assert_array_equal(ranges.astype(np.int64), o["ranges"])


def test_empty_and_fully_culled_scenes(gs):
    native, model = gs
    cam = scenes.identity_camera(40, 24, 30.0, bg=(0.1, 0.2, 0.3))
    s = scenes.tiny()
    s.means[2, :] = -1.0  # every Gaussian behind the camera
    run = DeviceRun(native, model, s, cam)
    assert run.K == 0
    img = host(run.image)
    for c in range(3):
        np.testing.assert_array_equal(img[c], np.float32(cam.bg[c]))
    np.testing.assert_array_equal(host(run.T), 1.0)
    np.testing.assert_array_equal(host(run.nc), 0)
    # backward of an empty render is zero and must not fault
    grads, _ = run.backward(np.ones((3, 24, 40)))
    for v in grads.values():
        assert not v.any()


def test_capacity_overflow_is_reported(gs):
    native, model = gs
    s = scenes.tiny()
    m = model.GaussianModel(s)
    cam = s.cameras[0]
    cs = native.camera_struct(cam)
    ctx = native.Context(s.n_pad, 8, cam.width, cam.height)
    ctx.preprocess(m.params_struct(), cs)
    img = torch.empty((3, 64, 64), device="cuda")
    T = torch.empty((64, 64), device="cuda")
    nc = torch.empty((64, 64), dtype=torch.int32, device="cuda")
    with pytest.raises(native.GsError) as e:
        ctx.render_forward(cs, img, T, nc)
    assert e.value.status == native.GS_ERR_CAPACITY
    # the context stays usable once the capacity is large enough
    ctx2 = native.Context(s.n_pad, 4096, cam.width, cam.height)
    ctx2.preprocess(m.params_struct(), cs)
    assert ctx2.render_forward(cs, img, T, nc) > 8


def test_invalid_arguments_are_rejected_on_the_host(gs):
    native, model = gs
    s = scenes.tiny()
    m = model.GaussianModel(s)
    ctx = native.Context(s.n_pad, 4096, 64, 64)
    cs = native.camera_struct(s.cameras[0])
    p = m.params_struct()
    p.n_pad = p.n_pad + 1
    with pytest.raises(native.GsError) as e:
        ctx.preprocess(p, cs)
    assert e.value.status == native.GS_ERR_INVALID_ARG
    p = m.params_struct()
    p.active_degree = 2
    with pytest.raises(native.GsError):
        ctx.preprocess(p, cs)
    big = native.camera_struct(scenes.identity_camera(65, 64, 64.0))
    with pytest.raises(native.GsError):
        ctx.preprocess(m.params_struct(), big)
    img = torch.empty((3, 64, 64), device="cuda")
    with pytest.raises(native.GsError):  # forward before preprocess
        native.Context(s.n_pad, 4096, 64, 64).render_forward(cs, img, img[0], img[0].int())


@pytest.mark.parametrize("shape", [(256, 256), (37, 45), (70, 33), (300, 97), (1, 40), (7, 3), (129, 64)])
def test_loss_matches_oracle(gs, shape):
    native, _ = gs
    H, W = shape
    rng = np.random.default_rng(H * 1000 + W)
    x = rng.uniform(0, 1, (3, H, W)).astype(np.float32)
    y = np.clip(x + rng.normal(0, 0.15, x.shape), 0, 1).astype(np.float32)
    x[:, :3, :5] = y[:, :3, :5]  # exact zero residuals: zero L1 subgradient
    ctx = native.Context(16, 16, W, H)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    d = torch.empty((3, H, W), device="cuda")
    ctx.loss_l1_dssim(dev(x), dev(y), 0.2, out, d)
    torch.cuda.synchronize()
    L, l1, ssim, dref = oracle.loss(x, y, 0.2)
    got = host(out)
    assert got[0] == pytest.approx(L, rel=LOSS_RTOL)
    assert got[1] == pytest.approx(l1, rel=LOSS_RTOL)
    assert got[2] == pytest.approx(ssim, rel=LOSS_RTOL, abs=1e-7)
    assert rel_l2(host(d), dref) < 1e-4
    # twice in a row gives the same value (deterministic reduction, counter reset)
    ctx.loss_l1_dssim(dev(x), dev(y), 0.2, out, d)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(out), got)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_backward_matches_oracle(gs, name):
    native, model = gs
    s, ci = SCENES[name]()
    cam = s.cameras[ci]
    run = DeviceRun(native, model, s, cam)
    r = run.oracle.render()
    target = scenes.uniform_image(cam.height, cam.width, seed=7)
    _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    dimg32 = dimg.astype(np.float32)
    ref = run.oracle.backward(dimg32.astype(np.float64))
    grads, sg = run.backward(dimg32)
    n = s.n
    vis = run.oracle.preprocess()["touched"] > 0
    assert rel_l2(sg[vis], ref["screen"][vis]) < GRAD_RL2
    for k in scenes.GROUP_NAMES:
        e = rel_l2(grads[k][..., :n], ref[k][..., :n])
        assert e < GRAD_RL2, (k, e)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_camera_gradient_matches_oracle(gs, name):
    """The pose gradient (dL/dw, dL/dt) the backward writes when
    gs_set_camera_grad is on, against the oracle's exact derivative, for the
    same dL/dimage."""
    native, model = gs
    s, ci = SCENES[name]()
    cam = s.cameras[ci]
    run = DeviceRun(native, model, s, cam)
    r = run.oracle.render()
    target = scenes.uniform_image(cam.height, cam.width, seed=8)
    _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    dimg32 = dimg.astype(np.float32)
    ref = run.oracle.camera_backward(run.oracle.backward(dimg32.astype(np.float64))["screen"])
    out = torch.full((6,), float("nan"), dtype=torch.float64, device="cuda")
    run.ctx.set_camera_grad(out)
    run.backward(dimg32)
    got = host(out)
    assert np.abs(ref).max() > 0
    assert rel_l2(got[:3], ref[:3]) < GRAD_RL2, (got, ref)
    assert rel_l2(got[3:], ref[3:]) < GRAD_RL2, (got, ref)


def test_camera_gradient_is_reproducible_and_the_same_on_the_fused_path(gs):
    """With fixed-point screen sums the pose gradient is bitwise the same on the
    separate and the fused backward (it is taken before the fused update), and
    run to run; with the output unset the backward no longer writes it."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    tgt = dev(scenes.uniform_image(cam.height, cam.width, seed=13))
    outs = []
    for fused in (False, True, True):
        m = model.GaussianModel(s)
        st = model.TrainStep(m, 200_000, cam.width, cam.height, fused_adam=fused, deterministic=True)
        out = torch.zeros(6, dtype=torch.float64, device="cuda")
        st.ctx.set_camera_grad(out)
        st(cam, tgt)
        torch.cuda.synchronize()
        outs.append(host(out).copy())
        st.ctx.set_camera_grad(None)
        out.fill_(7.0)
        st(cam, tgt)
        torch.cuda.synchronize()
        assert (host(out) == 7.0).all()
    assert np.abs(outs[0]).max() > 0
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[1], outs[2])


def test_adam_matches_oracle(gs):
    native, _ = gs
    rng = np.random.default_rng(11)
    n = 1003  # a ragged tail after the float4 body
    p = rng.normal(0, 1, n).astype(np.float32)
    m = rng.normal(0, 1e-3, n).astype(np.float32)
    v = rng.uniform(0, 1e-5, n).astype(np.float32)
    g = rng.normal(0, 1e-2, n).astype(np.float32)
    tp, tg, tm, tv = dev(p), dev(g), dev(m), dev(v)
    for step in (1, 7):
        native.adam_step(tp, tg, tm, tv, 1e-3, step)
        torch.cuda.synchronize()
        # the kernel receives lr, betas and eps as float32: give the oracle the same values
        f32 = lambda x: float(np.float32(x))
        rp, rg, rm, rv = oracle.adam(p, g, m, v, f32(1e-3), step, f32(0.9), f32(0.999), f32(1e-8))
        # float32 bound of b m + (1 - b) g: a few ulp of the two terms' magnitudes
        # (m itself can be much smaller than either term after cancellation)
        m_scale = 0.9 * np.abs(m) + 0.1 * np.abs(g)
        v_scale = 0.999 * np.abs(v) + 0.001 * g.astype(np.float64) ** 2
        assert np.all(np.abs(host(tm) - rm) <= 4e-7 * m_scale + 1e-30)
        assert np.all(np.abs(host(tv) - rv) <= 4e-7 * v_scale + 1e-30)
        # p moves by about lr per step; check the move to 1e-3 of lr
        dp = np.abs(host(tp) - rp)
        bad = dp > 1e-6 + 2e-7 * np.abs(rp)
        assert not bad.any(), (step, int(bad.sum()), float(dp.max()), int(np.argmax(dp)),
                               p[np.argmax(dp)], host(tp)[np.argmax(dp)], rp[np.argmax(dp)])
        assert not host(tg).any()
        p, m, v = host(tp), host(tm), host(tv)
        g = rng.normal(0, 1e-2, n).astype(np.float32)
        tg.copy_(dev(g))


@pytest.mark.parametrize("fused", [True, False])
def test_full_training_step_matches_oracle(gs, fused):
    """One iteration through model.TrainStep against the oracle's render -> loss ->
    backward -> Adam on the Small scene, with the backward and Adam either fused in
    one pass (gs_render_backward_adam) or as gs_render_backward + gs_adam_step."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    target = scenes.uniform_image(cam.height, cam.width, seed=9)
    m = model.GaussianModel(s)
    step = model.TrainStep(m, 200_000, cam.width, cam.height, fused_adam=fused)
    loss = step(cam, dev(target))
    torch.cuda.synchronize()
    o = oracle.Oracle(s, cam)
    r = o.render()
    L, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    assert host(loss)[0] == pytest.approx(L, rel=LOSS_RTOL)
    ref = o.backward(dimg)
    for k in scenes.GROUP_NAMES:
        p0 = getattr(s, k).astype(np.float64)
        rp, _, _, _ = oracle.adam(p0, ref[k], np.zeros_like(p0), np.zeros_like(p0), 1e-3, 1)
        got = host(m.params[k]).astype(np.float64)
        # the step is lr * sign-like; compare the update where the gradient is not tiny
        upd_ref = (rp.reshape(p0.shape) - p0)[..., : s.n]
        upd = (got - p0)[..., : s.n]
        big = np.abs(ref[k][..., : s.n]) > 1e-3 * np.abs(ref[k][..., : s.n]).max()
        frac = np.mean(np.abs(upd[big] - upd_ref[big]) <= 1e-6)
        assert frac > 0.99, (k, frac)


def test_fused_backward_adam_equals_separate_calls(gs):
    """Two iterations (with gradient accumulation left over between calls on the
    separate path's buffers) agree between the fused pass and the separate calls
    up to the float32 atomics' summation order; the fused pass zeroes the
    gradients and leaves invisible Gaussians moving by their moments only."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    tgt = dev(scenes.uniform_image(cam.height, cam.width, seed=12))
    runs = []
    for fused in (False, True):
        m = model.GaussianModel(s)
        st = model.TrainStep(m, 200_000, cam.width, cam.height, fused_adam=fused)
        for _ in range(2):
            st(cam, tgt)
        torch.cuda.synchronize()
        assert not m.grad_flat.any().item()
        runs.append(m)
    a, b = runs
    for k in scenes.GROUP_NAMES:
        np.testing.assert_allclose(host(a.m[k]), host(b.m[k]), rtol=1e-3, atol=1e-9)
        np.testing.assert_allclose(host(a.v[k]), host(b.v[k]), rtol=2e-3, atol=1e-13)
        dp = np.abs(host(a.params[k]) - host(b.params[k]))
        assert np.mean(dp <= 1e-6) > 0.999, k


def test_fused_backward_adam_adds_an_accumulated_gradient(gs):
    """With a gradient buffer, the fused pass adds the accumulated gradient to
    this view's before the update (and zeroes it): a render_backward of a first
    loss gradient followed by the fused pass of a second equals two
    render_backward calls followed by gs_adam_step on every group, up to the
    float32 atomics' summation order."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    cs = native.camera_struct(cam)
    H, W = cam.height, cam.width
    rng = np.random.default_rng(17)
    d1 = dev(rng.normal(0, 1e-5, (3, H, W)))
    d2 = dev(rng.normal(0, 1e-5, (3, H, W)))
    runs = []
    for fused in (False, True):
        m = model.GaussianModel(s)
        st = model.TrainStep(m, 200_000, W, H, fused_adam=fused)
        _, T, nc = st.forward(cs, H, W)
        st.ctx.render_backward(m.params_struct(), cs, T, nc, d1, m.grads_struct())
        if fused:
            em, ev = m.moments_structs()
            st.ctx.render_backward_adam(m.params_struct(), cs, T, nc, d2, m.grads_struct(), em, ev,
                                        [1e-3] * 5, 1)
        else:
            st.ctx.render_backward(m.params_struct(), cs, T, nc, d2, m.grads_struct())
            for k in scenes.GROUP_NAMES:
                native.adam_step(m.params[k], m.grads[k], m.m[k], m.v[k], 1e-3, 1)
        torch.cuda.synchronize()
        assert not m.grad_flat.any().item()
        runs.append(m)
    a, b = runs
    for k in scenes.GROUP_NAMES:
        assert rel_l2(host(b.m[k]), host(a.m[k])) < 1e-4, k
        dp = np.abs(host(a.params[k]) - host(b.params[k]))
        assert np.mean(dp <= 1e-6) > 0.999, k


def test_a_second_backward_after_one_forward_starts_from_cleared_sums(gs):
    """The forward clears the screen-gradient sums for the backward; a second
    backward of the same forward must clear them itself, so both give the same
    gradient (up to the float32 atomics' summation order) instead of the second
    adding onto the first."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    cs = native.camera_struct(cam)
    H, W = cam.height, cam.width
    d = dev(np.random.default_rng(23).normal(0, 1e-5, (3, H, W)))
    m = model.GaussianModel(s)
    st = model.TrainStep(m, 200_000, W, H, fused_adam=False)
    _, T, nc = st.forward(cs, H, W)
    grads = []
    for _ in range(2):
        m.grad_flat.zero_()
        st.ctx.render_backward(m.params_struct(), cs, T, nc, d, m.grads_struct())
        torch.cuda.synchronize()
        grads.append(host(m.grad_flat).astype(np.float64))
    assert np.abs(grads[0]).max() > 0
    assert rel_l2(grads[1], grads[0]) < 1e-4


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_opacity_aware_rect_path_matches_oracle(gs, name):
    """With the opacity-aware tile rect: rects and the sort bit-exact, pixels
    and gradients within tolerance, against the oracle run with the same rect;
    fewer entries than the 3-sigma rect."""
    native, model = gs
    s, ci = SCENES[name]()
    cam = s.cameras[ci]
    run = DeviceRun(native, model, s, cam, opacity_rect=True)
    g = run.preprocess_out()
    o = run.oracle.preprocess()
    np.testing.assert_array_equal(g["touched"], o["touched"])
    vis = o["touched"] > 0
    np.testing.assert_array_equal(g["rect"][vis], o["rect"][vis])
    ids, tiles, ranges = run.sorted_out()
    srt = run.oracle.sorted()
    np.testing.assert_array_equal(ids, srt["ids"])
    np.testing.assert_array_equal(tiles, srt["tiles"])
    np.testing.assert_array_equal(ranges.astype(np.int64), srt["ranges"])
    assert run.K < DeviceRun(native, model, s, cam).K
    r = run.oracle.render()
    check_pixels(run, r)
    target = scenes.uniform_image(cam.height, cam.width, seed=7)
    _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    dimg32 = dimg.astype(np.float32)
    ref = run.oracle.backward(dimg32.astype(np.float64))
    grads, sg = run.backward(dimg32)
    assert rel_l2(sg[vis], ref["screen"][vis]) < GRAD_RL2
    for k in scenes.GROUP_NAMES:
        e = rel_l2(grads[k][..., :s.n], ref[k][..., :s.n])
        assert e < GRAD_RL2, (k, e)


@pytest.mark.parametrize("name,rect", [("tiny", False), ("small", False), ("small", True)])
def test_mip_compensation_path_matches_oracle(gs, name, rect):
    """With the Mip-Splatting compensation factor: the screen opacities, the
    pixels and every gradient against the oracle run with the factor; with the
    opacity-aware rect (which uses opacity * comp) also the rects and the sort,
    bit for bit. The factor changes the image by far more than the tolerance."""
    native, model = gs
    s, ci = SCENES[name]()
    cam = s.cameras[ci]
    run = DeviceRun(native, model, s, cam, opacity_rect=rect, mip_comp=True)
    g = run.preprocess_out()
    o = run.oracle.preprocess()
    np.testing.assert_array_equal(g["touched"], o["touched"])
    vis = o["touched"] > 0
    np.testing.assert_array_equal(g["rect"][vis], o["rect"][vis])
    np.testing.assert_allclose(g["opacity"][vis], o["screen"][vis, 5], rtol=3e-6, atol=1e-7)
    ids, tiles, ranges = run.sorted_out()
    srt = run.oracle.sorted()
    np.testing.assert_array_equal(ids, srt["ids"])
    np.testing.assert_array_equal(ranges.astype(np.int64), srt["ranges"])
    r = run.oracle.render()
    check_pixels(run, r)
    plain = oracle.Oracle(s, cam, opacity_rect=rect).render()
    assert np.abs(plain["image"] - r["image"]).max() > 1e-2
    target = scenes.uniform_image(cam.height, cam.width, seed=7)
    _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    dimg32 = dimg.astype(np.float32)
    ref = run.oracle.backward(dimg32.astype(np.float64))
    grads, sg = run.backward(dimg32)
    assert rel_l2(sg[vis], ref["screen"][vis]) < GRAD_RL2
    for k in scenes.GROUP_NAMES:
        e = rel_l2(grads[k][..., :s.n], ref[k][..., :s.n])
        assert e < GRAD_RL2, (k, e)


def test_mip_compensation_in_the_fused_training_step(gs):
    """One fused backward + Adam step with the factor against the oracle's
    backward and Adam on the same image gradient."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    run = DeviceRun(native, model, s, cam, mip_comp=True)
    r = run.oracle.render()
    target = scenes.uniform_image(cam.height, cam.width, seed=8)
    _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    dimg32 = dimg.astype(np.float32)
    ref = run.oracle.backward(dimg32.astype(np.float64))
    m = run.m
    p0 = {k: host(m.params[k]).astype(np.float64) for k in scenes.GROUP_NAMES}
    em, ev = m.moments_structs()
    lr = 1e-3
    run.ctx.render_backward_adam(m.params_struct(), run.cs, run.T, run.nc, torch.from_numpy(dimg32).cuda(),
                                 None, em, ev, [lr] * 5, 1, 0.9, 0.999, 1e-8)
    torch.cuda.synchronize()
    for k in scenes.GROUP_NAMES:
        want = oracle.adam(p0[k], ref[k], np.zeros_like(p0[k]), np.zeros_like(p0[k]), lr, 1)[0]
        got = host(m.params[k]).astype(np.float64).reshape(-1)
        # Adam's first step moves each scalar by lr sign(g) wherever |g| >> eps
        sel = np.abs(ref[k].reshape(-1)) > 1e-5 * np.abs(ref[k]).max()
        sel &= np.arange(got.size) % m.n_pad < s.n
        assert np.mean(np.abs(got[sel] - want[sel]) <= 1e-6) > 0.995, k


def test_set_option_rejects_unknown_options(gs):
    native, _ = gs
    ctx = native.Context(16, 16, 16, 16)
    with pytest.raises(native.GsError):
        ctx.set_option(99, 1)
    with pytest.raises(native.GsError):
        ctx.set_option(native.GS_OPTION_OPACITY_RECT, 2)


def test_deterministic_backward_is_bitwise_reproducible_and_matches_oracle(gs):
    """With GS_OPTION_DETERMINISTIC the screen-gradient sums are integer
    (fixed-point) atomics: two independent runs give the same bits, for the
    backward and for two fused training steps, and the gradients still match
    the oracle."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    target = scenes.uniform_image(cam.height, cam.width, seed=7)
    outs = []
    for _ in range(2):
        run = DeviceRun(native, model, s, cam)
        run.ctx.set_option(native.GS_OPTION_DETERMINISTIC, 1)
        run.ctx.preprocess(run.m.params_struct(), run.cs)
        run.K = run.ctx.render_forward(run.cs, run.image, run.T, run.nc)
        r = run.oracle.render()
        _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
        grads, sg = run.backward(dimg.astype(np.float32))
        outs.append((grads, sg, run))
    (g1, sg1, run), (g2, sg2, _) = outs
    np.testing.assert_array_equal(sg1.view(np.uint32), sg2.view(np.uint32))
    for k in scenes.GROUP_NAMES:
        np.testing.assert_array_equal(g1[k].view(np.uint32), g2[k].view(np.uint32))
    ref = run.oracle.backward(dimg.astype(np.float32).astype(np.float64))
    vis = run.oracle.preprocess()["touched"] > 0
    assert rel_l2(sg1[vis], ref["screen"][vis]) < GRAD_RL2
    for k in scenes.GROUP_NAMES:
        assert rel_l2(g1[k][..., :s.n], ref[k][..., :s.n]) < GRAD_RL2, k
    # two fused training steps, twice from the same start
    tgt = dev(target)
    params = []
    for _ in range(2):
        m = model.GaussianModel(s)
        st = model.TrainStep(m, 200_000, cam.width, cam.height, deterministic=True)
        for _ in range(2):
            st(cam, tgt)
        torch.cuda.synchronize()
        params.append(host(m.flat).view(np.uint32).copy())
    np.testing.assert_array_equal(params[0], params[1])


@pytest.mark.parametrize("shape", [(256, 256), (37, 45), (1, 5)])
def test_charbonnier_loss_matches_oracle(gs, shape):
    native, _ = gs
    H, W = shape
    rng = np.random.default_rng(H + W)
    x = rng.uniform(0, 1, (3, H, W)).astype(np.float32)
    y = np.clip(x + rng.normal(0, 0.2, x.shape), 0, 1).astype(np.float32)
    y[0, 0, 0] = 40.0  # an outlier
    gain, bias = [1.1, 0.9, 1.02], [0.03, -0.02, 0.0]
    ctx = native.Context(16, 16, max(W, 16), max(H, 16))
    out = torch.zeros(7, dtype=torch.float64, device="cuda")
    d = torch.empty((3, H, W), device="cuda")
    f32 = [float(np.float32(v)) for v in gain], [float(np.float32(v)) for v in bias]
    ctx.loss_charbonnier(dev(x), dev(y), gain, bias, out, d)
    torch.cuda.synchronize()
    L, dref, dg, db = oracle.charbonnier_loss(x, y, f32[0], f32[1])
    got = host(out)
    assert got[0] == pytest.approx(L, rel=LOSS_RTOL)
    np.testing.assert_allclose(got[1:4], dg, rtol=1e-5, atol=1e-9)
    np.testing.assert_allclose(got[4:7], db, rtol=1e-5, atol=1e-9)
    assert rel_l2(host(d), dref) < 1e-5
    ctx.loss_charbonnier(dev(x), dev(y), gain, bias, out, d)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(out), got)  # deterministic, counter reset


def test_training_step_with_the_charbonnier_loss(gs):
    """One TrainStep iteration with the Charbonnier loss: its loss value is the
    oracle's for the same render, and the update moves parameters as the
    oracle's backward + Adam of that loss does."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    target = scenes.uniform_image(cam.height, cam.width, seed=9)
    m = model.GaussianModel(s)
    step = model.TrainStep(m, 200_000, cam.width, cam.height, loss="charbonnier")
    loss = step(cam, dev(target))
    torch.cuda.synchronize()
    o = oracle.Oracle(s, cam)
    r = o.render()
    L, dimg, _, _ = oracle.charbonnier_loss(r["image"].astype(np.float32), target, [1, 1, 1], [0, 0, 0])
    assert host(loss)[0] == pytest.approx(L, rel=1e-4)
    ref = o.backward(dimg)
    for k in scenes.GROUP_NAMES:
        p0 = getattr(s, k).astype(np.float64)
        rp, _, _, _ = oracle.adam(p0, ref[k], np.zeros_like(p0), np.zeros_like(p0), 1e-3, 1)
        upd_ref = (rp.reshape(p0.shape) - p0)[..., : s.n]
        upd = (host(m.params[k]).astype(np.float64) - p0)[..., : s.n]
        big = np.abs(ref[k][..., : s.n]) > 1e-3 * np.abs(ref[k][..., : s.n]).max()
        assert np.mean(np.abs(upd[big] - upd_ref[big]) <= 1e-6) > 0.99, k


def test_sh_degree_ramp_leaves_inactive_bands_untouched(gs):
    """TrainStep(sh_ramp_every=2): degree 0 for the first two iterations (the
    higher SH bands neither colour nor move), then degree 1 (bands 1-3 move,
    bands 4-15 still do not)."""
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    tgt = dev(scenes.uniform_image(cam.height, cam.width, seed=14))
    m = model.GaussianModel(s)
    st = model.TrainStep(m, 200_000, cam.width, cam.height, sh_ramp_every=2)
    sh0 = host(m.params["sh"]).copy()
    st(cam, tgt)
    st(cam, tgt)
    torch.cuda.synchronize()
    assert m.active_degree == 0
    sh1 = host(m.params["sh"]).copy()
    np.testing.assert_array_equal(sh1[:, 1:], sh0[:, 1:])
    assert not np.array_equal(sh1[:, 0], sh0[:, 0])
    st(cam, tgt)
    torch.cuda.synchronize()
    assert m.active_degree == 1
    sh2 = host(m.params["sh"])
    np.testing.assert_array_equal(sh2[:, 4:], sh0[:, 4:])
    assert not np.array_equal(sh2[:, 1:4], sh0[:, 1:4])
