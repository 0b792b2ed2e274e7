"""Parity at full size: the Mid workload (500,000 Gaussians, 1280x720), the
Dense workload (3,000,000 Gaussians, SH degree 3, 1920x1080) and the
Heavy-tail workload (6,000,000 Gaussians, 10% of them large, so long per-tile
lists) in the launch configuration the benchmark times (one TrainStep with its
entry capacity), against the float64 oracle.

The oracle's preprocess and tile sort run on the whole scene, so those are
compared in full (the sort bit-exact over every entry). The blend is compared
on sampled pixels (random ones, plus every pixel of a corner tile, an interior
tile and a tile of the ragged last tile row: 1080 = 67.5 tiles), which the
oracle walks one by one; a pixel whose walk meets a decision within float32
reach of its threshold must equal one of the oracle's replays of the walk
with such decisions taken either way. The loss is compared in full. The backward and the
fused backward + Adam are compared for a loss gradient restricted to a band
of 16 pixel rows: the oracle runs the blend backward of those rows and the
projection backward of every Gaussian, and the property that rows outside the
band contribute nothing holds at any size.
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
BAND = 16
MIN_UNAMBIGUOUS = {"mid": 0.99, "dense": 0.99, "heavy_tail": 0.95}
REPLAY_BITS = 6  # ambiguous decisions per pixel whose 2^k replays are all tried


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    return t.detach().cpu().numpy()


def rel_l2(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


@pytest.fixture(scope="module", params=["mid", "dense", "heavy_tail"])
def full(request):
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import model, native
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    native.load()
    scene = scenes.CONFIGS[request.param]()
    cams = scene.cameras
    cam = cams[int(scenes.camera_schedule(len(cams), 1, seed=0)[0])]
    m = model.GaussianModel(scene)
    W = max(c.width for c in cams)
    H = max(c.height for c in cams)
    step = model.TrainStep(m, max(1 << 20, 8 * scene.n), W, H)
    cs = native.camera_struct(cam)
    img, T, nc = step.forward(cs, cam.height, cam.width)
    torch.cuda.synchronize()
    o = oracle.Oracle(scene, cam)
    return dict(native=native, model=model, scene=scene, cam=cam, m=m, step=step, cs=cs,
                img=img, T=T, nc=nc, o=o)


def test_full_preprocess_and_sort_bit_exact(full):
    step, o, n = full["step"], full["o"], full["scene"].n
    out = dict(rect=torch.empty((n, 4), dtype=torch.int32, device="cuda"),
               touched=torch.empty(n, dtype=torch.int32, device="cuda"),
               depth=torch.empty(n, device="cuda"), mean2d=torch.empty((n, 2), device="cuda"))
    step.ctx.debug_preprocess(**out)
    torch.cuda.synchronize()
    g = {k: host(v) for k, v in out.items()}
    pp = o.preprocess()
    np.testing.assert_array_equal(g["touched"], pp["touched"])
    vis = pp["touched"] > 0
    assert vis.sum() > n // 2
    np.testing.assert_array_equal(g["rect"][vis], pp["rect"][vis])
    np.testing.assert_array_equal(g["depth"].view(np.uint32)[vis], pp["depth_key"].view(np.uint32)[vis])
    np.testing.assert_allclose(g["mean2d"][vis], pp["screen"][vis, 0:2], rtol=0, atol=1e-3)

    srt = o.sorted()
    K = step.last_entries
    assert K == srt["ids"].size
    cam = full["cam"]
    tx, ty = (cam.width + 15) // 16, (cam.height + 15) // 16
    ids = torch.empty(K, dtype=torch.int32, device="cuda")
    tiles = torch.empty(K, dtype=torch.int32, device="cuda")
    ranges = torch.empty((tx * ty, 2), dtype=torch.int32, device="cuda")
    step.ctx.debug_sorted(ids, tiles, ranges)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(ids), srt["ids"])
    np.testing.assert_array_equal(host(tiles), srt["tiles"])
    np.testing.assert_array_equal(host(ranges).astype(np.int64), srt["ranges"])


def sample_pixels(cam, seed=5, n_random=4096):
    rng = np.random.default_rng(seed)
    px = [rng.integers(0, cam.width, n_random)]
    py = [rng.integers(0, cam.height, n_random)]
    tx, ty = (cam.width + 15) // 16, (cam.height + 15) // 16
    for t_x, t_y in ((0, 0), (tx // 2, ty // 2), (tx - 1, ty - 1), (tx // 3, ty - 1)):
        ys, xs = np.mgrid[16 * t_y:min(16 * t_y + 16, cam.height), 16 * t_x:min(16 * t_x + 16, cam.width)]
        px.append(xs.ravel())
        py.append(ys.ravel())
    return np.concatenate(px), np.concatenate(py)


def test_full_forward_sampled_pixels(full):
    cam, o = full["cam"], full["o"]
    px, py = sample_pixels(cam)
    r = o.render_pixels(px, py)
    img, T, nc = host(full["img"]), host(full["T"]), host(full["nc"])
    ok = ~r["ambiguous"].astype(bool)
    # pixels with a threshold decision within 1e-6 relative of its cut are left out:
    # the longer the lists (thousands per tile on Heavy-tail), the more of them
    assert ok.mean() > MIN_UNAMBIGUOUS[full["scene"].name], ok.mean()
    got = img[:, py, px].T
    err = np.abs(got - r["rgb"])[ok]
    assert err.max() <= PIX_TOL, err.max()
    # T enters the pixel as T * background: compared at the pixel tolerance
    np.testing.assert_allclose(T[py, px][ok], r["T"][ok], rtol=0, atol=PIX_TOL)
    np.testing.assert_array_equal(nc[py, px][ok], r["n_contrib"][ok])
    # Every ambiguous pixel must equal one of the oracle's replays of its walk with
    # some of its near-threshold decisions taken the other way (a float32 renderer
    # may take each of them either way): all pixels with up to REPLAY_BITS such
    # decisions are checked; pixels with more must stay rare.
    amb = np.nonzero(~ok)[0]
    matched = np.zeros(amb.size, bool)
    n_amb = o.replay_pixels(px[amb], py[amb], 0)["n_amb"]
    bits = int(min(REPLAY_BITS, n_amb.max(initial=0)))
    for mask in range(1 << bits):
        rep = o.replay_pixels(px[amb], py[amb], mask)
        matched |= ((np.abs(got[~ok] - rep["rgb"]).max(axis=1) <= PIX_TOL) &
                    (np.abs(T[py, px][~ok] - rep["T"]) <= PIX_TOL) & (nc[py, px][~ok] == rep["n_contrib"]))
    enumerable = n_amb <= REPLAY_BITS
    assert matched[enumerable].all(), (np.nonzero(~matched[enumerable])[0][:10], n_amb[~matched][:10])
    assert (~enumerable).sum() <= 0.005 * px.size, (~enumerable).sum()
    # properties that hold at every pixel
    assert np.all((T >= 0) & (T <= 1))
    assert np.all(nc >= 0)


def band_gradient(full):
    """The loss gradient of the full image against a uniform target, kept on a
    16-row band through the image centre and zero elsewhere."""
    cam = full["cam"]
    H, W = cam.height, cam.width
    target = scenes.uniform_image(H, W, seed=21)
    img32 = host(full["img"])
    L, l1, ssim, d = oracle.loss(img32, target, 0.2)
    y0 = (H - BAND) // 2
    band = np.zeros((3, H, W), np.float32)
    band[:, y0:y0 + BAND, :] = d[:, y0:y0 + BAND, :]
    return target, (L, l1, ssim, d), band, y0


def test_full_loss_full_image(full):
    step = full["step"]
    target, (L, l1, ssim, dref), _, _ = band_gradient(full)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    d = torch.empty_like(full["img"])
    step.ctx.loss_l1_dssim(full["img"], dev(target), 0.2, out, d)
    torch.cuda.synchronize()
    got = host(out)
    assert got[0] == pytest.approx(L, rel=LOSS_RTOL)
    assert got[1] == pytest.approx(l1, rel=LOSS_RTOL)
    assert got[2] == pytest.approx(ssim, rel=LOSS_RTOL, abs=1e-7)
    assert rel_l2(host(d), dref) < 1e-4


def oracle_band_backward(full, band, y0):
    o, s = full["o"], full["scene"]
    sg = np.zeros((s.n, 9))
    o.blend_backward_rows(y0, y0 + BAND, band.astype(np.float64), sg)
    out = dict(means=np.zeros((3, s.n_pad)), log_scales=np.zeros((3, s.n_pad)),
               quats=np.zeros((4, s.n_pad)), opacity_logits=np.zeros(s.n_pad),
               sh=np.zeros((3, s.sh_k, s.n_pad)))
    o.project_backward(sg, 0, s.n, out)
    return sg, out


def test_full_backward_on_a_row_band(full):
    step, m, s = full["step"], full["m"], full["scene"]
    _, _, band, y0 = band_gradient(full)
    sg_ref, ref = oracle_band_backward(full, band, y0)
    m.grad_flat.zero_()
    cam_grad = torch.zeros(6, dtype=torch.float64, device="cuda")
    step.ctx.set_camera_grad(cam_grad)
    step.ctx.render_backward(m.params_struct(), full["cs"], full["T"], full["nc"], dev(band),
                             m.grads_struct())
    step.ctx.set_camera_grad(None)
    sg = torch.empty((s.n, 9), device="cuda")
    step.ctx.debug_screen_grads(sg)
    torch.cuda.synchronize()
    sg = host(sg)
    assert np.any(sg_ref != 0, axis=1).sum() > 1000
    # a Gaussian none of whose tiles meets the band's tile rows gets exactly nothing
    rect = full["o"].preprocess()["rect"]  # x0, y0, x1, y1 in tiles
    far = (rect[:, 3] < y0 // 16) | (rect[:, 1] > (y0 + BAND - 1) // 16)
    assert not sg[far].any(), "Gaussians away from the band got a screen gradient"
    assert rel_l2(sg, sg_ref) < GRAD_RL2
    for k in scenes.GROUP_NAMES:
        e = rel_l2(host(m.grads[k])[..., :s.n], ref[k][..., :s.n])
        assert e < GRAD_RL2, (k, e)
    # the camera-pose gradient of the same band
    cam_ref = full["o"].camera_backward(sg_ref)
    got = host(cam_grad)
    assert rel_l2(got[:3], cam_ref[:3]) < GRAD_RL2, (got, cam_ref)
    assert rel_l2(got[3:], cam_ref[3:]) < GRAD_RL2, (got, cam_ref)
    m.grad_flat.zero_()


def test_full_fused_backward_adam_on_a_row_band(full):
    step, m, s = full["step"], full["m"], full["scene"]
    _, _, band, y0 = band_gradient(full)
    _, ref = oracle_band_backward(full, band, y0)
    m.load(s)
    m.m_flat.zero_()
    m.v_flat.zero_()
    m.grad_flat.zero_()
    em, ev = m.moments_structs()
    lr = 1e-3
    step.ctx.render_backward_adam(m.params_struct(), full["cs"], full["T"], full["nc"], dev(band),
                                  None, em, ev, [lr] * 5, 1)
    torch.cuda.synchronize()
    assert not m.grad_flat.any().item()
    f32 = lambda x: float(np.float32(x))
    for k in scenes.GROUP_NAMES:
        p0 = getattr(s, k).astype(np.float64)[..., :s.n]
        g = ref[k][..., :s.n]
        rp, _, rm, _ = oracle.adam(p0, g, np.zeros_like(p0), np.zeros_like(p0),
                                    f32(lr), 1, f32(0.9), f32(0.999), f32(1e-8))
        got = host(m.params[k]).astype(np.float64)[..., :s.n]
        # untouched Gaussians (zero gradient, zero moments) do not move at all
        zero = g == 0
        np.testing.assert_array_equal(got[zero], p0[zero].astype(np.float32))
        # at step 1 the update is lr * g / (|g| + eps'): compare where the gradient is not tiny
        big = np.abs(g) > 1e-3 * np.abs(g).max()
        frac = np.mean(np.abs((got - p0)[big] - (rp.reshape(p0.shape) - p0)[big]) <= 1e-6)
        assert frac > 0.99, (k, frac)
        assert rel_l2(host(m.m[k])[..., :s.n], rm.reshape(p0.shape)) < GRAD_RL2, k
    m.load(s)
    m.m_flat.zero_()
    m.v_flat.zero_()


def test_full_image_backward_at_mid(full):
    """The blend and projection backward of the whole image's loss gradient (not a
    band) at Mid, where the float64 oracle can walk every pixel: its row bands run
    on the host's cores at once (its calls only read the shared scene state), each
    band into a screen-gradient buffer of its own, summed in band order. Exercises
    every tile and the atomics contention of a full-image gradient."""
    if full["scene"].name != "mid":
        pytest.skip("the oracle's full-image backward is timed for the Mid workload")
    import concurrent.futures
    import os
    step, m, s, o = full["step"], full["m"], full["scene"], full["o"]
    cam = full["cam"]
    H = cam.height
    _, (_, _, _, d), _, _ = band_gradient(full)
    d64 = d.astype(np.float32).astype(np.float64)
    nb = max(1, min(len(os.sched_getaffinity(0)), 32))
    edges = np.linspace(0, H, nb + 1).astype(int)
    bufs = [np.zeros((s.n, 9)) for _ in range(nb)]
    with concurrent.futures.ThreadPoolExecutor(nb) as ex:
        list(ex.map(lambda k: o.blend_backward_rows(edges[k], edges[k + 1], d64, bufs[k]), range(nb)))
    sg_ref = np.sum(bufs, axis=0)
    ref = dict(means=np.zeros((3, s.n_pad)), log_scales=np.zeros((3, s.n_pad)), quats=np.zeros((4, s.n_pad)),
               opacity_logits=np.zeros(s.n_pad), sh=np.zeros((3, s.sh_k, s.n_pad)))
    cuts = np.linspace(0, s.n, nb + 1).astype(int)
    with concurrent.futures.ThreadPoolExecutor(nb) as ex:
        list(ex.map(lambda k: o.project_backward(sg_ref, cuts[k], cuts[k + 1], ref), range(nb)))
    m.grad_flat.zero_()
    step.ctx.render_backward(m.params_struct(), full["cs"], full["T"], full["nc"], dev(d.astype(np.float32)),
                             m.grads_struct())
    sg = torch.empty((s.n, 9), device="cuda")
    step.ctx.debug_screen_grads(sg)
    torch.cuda.synchronize()
    sg = host(sg)
    touched = o.preprocess()["touched"] > 0
    assert np.any(sg_ref[touched] != 0, axis=1).mean() > 0.5
    assert not sg[~touched].any()
    assert rel_l2(sg, sg_ref) < GRAD_RL2
    for k in scenes.GROUP_NAMES:
        e = rel_l2(host(m.grads[k])[..., :s.n], ref[k][..., :s.n])
        assert e < GRAD_RL2, (k, e)
    m.grad_flat.zero_()
