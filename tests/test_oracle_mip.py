"""The oracle's Mip-Splatting compensation factor (off by default) against what
fixes it: the pages apply it as alpha = min(0.99, opacity * comp * exp(-e)) and
in the opacity-aware radius ("How a computer rebuilds a real place ... Gaussian
Splats", section "Flattening a 3D blob into a 2D oval (EWA projection)"), and
Mip-Splatting's 2D filter defines it as sqrt(det V / det(V + s I)) with s the
0.3 px^2 dilation. Pinned by the closed form of an isotropic splat on the
optical axis, its limits, the integrated weight of an anisotropic splat (which
the factor makes equal to the undilated splat's, by quadrature), the default
path being unchanged, and central differences of the rendered loss."""
import math

import numpy as np
import pytest
from scipy.spatial.transform import Rotation

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes

DILATION = 0.3


def one_gaussian(z, scales, quat=(1.0, 0.0, 0.0, 0.0), logit=0.4, W=64, H=64, f=64.0):
    cam = scenes.identity_camera(W, H, f)
    means = np.array([[0.0], [0.0], [z]])
    ls = np.log(np.asarray(scales, np.float64)).reshape(3, 1)
    q = np.asarray(quat, np.float64).reshape(4, 1)
    sh = np.ones((3, 1, 1))
    return scenes.make_scene("mip", means, ls, q, np.array([logit]), 0, sh, [cam], dtype=np.float64), cam


def sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


@pytest.mark.parametrize("sigma,z", [(0.002, 4.0), (0.01, 3.0), (0.05, 5.0), (0.3, 2.0)])
def test_isotropic_splat_on_the_axis_closed_form(sigma, z):
    """On the optical axis with the identity pose, J W = (f / z) [I | 0], so an
    isotropic splat has V = v I with v = (f sigma / z)^2 and comp = v / (v + 0.3).
    The centre pixel's alpha (e = 0) is then the opacity times comp."""
    logit = 0.4
    s, cam = one_gaussian(z, (sigma,) * 3, logit=logit)
    v = (cam.fx * sigma / z) ** 2
    comp = v / (v + DILATION)
    o = oracle.Oracle(s, cam, mip_comp=True)
    pp = o.preprocess()
    assert pp["screen"][0, 5] == pytest.approx(sigmoid(logit) * comp, rel=1e-12)
    img = o.render()["image"]
    alpha = sigmoid(logit) * comp
    cx, cy = int(cam.cx), int(cam.cy)  # the mean projects exactly onto pixel (32, 32)
    if alpha >= 1 / 255:
        assert img[0, cy, cx] == pytest.approx(alpha, rel=1e-12)
    else:
        assert img[0, cy, cx] == 0.0  # below the alpha floor the splat is skipped
    # without the option the same splat keeps its plain opacity
    plain = oracle.Oracle(s, cam).preprocess()
    assert plain["screen"][0, 5] == pytest.approx(sigmoid(logit), rel=1e-15)


def test_factor_tends_to_one_for_large_splats_and_zero_for_tiny_ones():
    comps = []
    for sigma in (1e-4, 1e-3, 1e-2, 1e-1, 1.0):
        s, cam = one_gaussian(3.0, (sigma, 1.3 * sigma, 0.8 * sigma), quat=(0.9, 0.2, -0.3, 0.1))
        o = oracle.Oracle(s, cam, mip_comp=True).preprocess()
        comps.append(o["screen"][0, 5] / sigmoid(0.4))
    assert all(0.0 < c <= 1.0 for c in comps)
    assert all(a < b for a, b in zip(comps, comps[1:]))  # grows with the splat
    assert comps[0] < 1e-4 and comps[-1] > 0.999


def test_compensated_splat_keeps_the_undilated_weight():
    """The integral of o comp exp(-e) over the screen (quadrature on a 0.02 px grid
    of the oracle's screen record) equals the weight of the undilated splat,
    2 pi o sqrt(det V). V is computed here independently: on the optical axis
    with the identity pose V = (f / z)^2 times the upper-left 2 x 2 block of
    Sigma = R S^2 R^T, with R from scipy's rotation."""
    z, scales, quat, logit = 3.0, (0.006, 0.02, 0.011), (0.8, 0.3, -0.4, 0.2), 0.4
    s, cam = one_gaussian(z, scales, quat=quat, logit=logit)
    R = Rotation.from_quat([quat[1], quat[2], quat[3], quat[0]]).as_matrix()
    Sigma = R @ np.diag(np.square(scales)) @ R.T
    V = (cam.fx / z) ** 2 * Sigma[:2, :2]
    pp = oracle.Oracle(s, cam, mip_comp=True).preprocess()
    u, v, A, B, C, o_eff = pp["screen"][0, :6]
    h = 0.02
    xs = np.arange(-12.0, 12.0, h) + h / 2
    dx, dy = np.meshgrid(xs, xs, indexing="xy")
    e = 0.5 * (A * dx * dx + C * dy * dy) + B * dx * dy
    weight = o_eff * np.exp(-e).sum() * h * h
    assert weight == pytest.approx(2 * math.pi * sigmoid(logit) * math.sqrt(np.linalg.det(V)), rel=1e-6)
    # without the factor the dilated splat carries more weight than the undilated one
    pp0 = oracle.Oracle(s, cam).preprocess()
    u0, v0, A0, B0, C0, o0 = pp0["screen"][0, :6]
    w0 = o0 * np.exp(-(0.5 * (A0 * dx * dx + C0 * dy * dy) + B0 * dx * dy)).sum() * h * h
    assert w0 > 1.5 * weight


def test_default_path_is_unchanged_and_tile_lists_shrink_only_with_the_opacity_rect():
    s = scenes.small()
    cam = s.cameras[0]
    a, b = oracle.Oracle(s, cam), oracle.Oracle(s, cam, mip_comp=True)
    pa, pb = a.preprocess(), b.preprocess()
    # geometry, colour and the 3-sigma tile lists do not depend on the factor
    for k in ("cov2d", "depth", "rect", "touched"):
        np.testing.assert_array_equal(pa[k], pb[k])
    np.testing.assert_array_equal(pa["screen"][:, [0, 1, 2, 3, 4, 6, 7, 8]], pb["screen"][:, [0, 1, 2, 3, 4, 6, 7, 8]])
    vis = pa["touched"] > 0
    ratio = pb["screen"][vis, 5] / pa["screen"][vis, 5]
    assert np.all((ratio > 0) & (ratio <= 1.0))
    # the opacity-aware radius uses opacity * comp: never more tiles than without it
    ra, rb = oracle.Oracle(s, cam, opacity_rect=True), oracle.Oracle(s, cam, opacity_rect=True, mip_comp=True)
    ta, tb = ra.preprocess()["touched"], rb.preprocess()["touched"]
    assert np.all(tb <= ta) and tb.sum() < ta.sum()


def _gc_scene(seed):
    rng = np.random.default_rng(seed)
    n = 12
    means = np.stack([rng.uniform(-0.6, 0.6, n), rng.uniform(-0.45, 0.45, n), rng.uniform(2.0, 4.0, n)])
    # small splats, a few pixels across, where the factor is far from 1
    ls = rng.normal(math.log(0.02), 0.3, (3, n))
    q = rng.normal(size=(4, n))
    logits = rng.normal(1.0, 1.0, n)
    sh = np.zeros((3, 16, n))
    sh[:, 0] = rng.uniform(0.3, 1.0, (3, n))
    sh[:, 1:] = rng.normal(0.0, 0.3, (3, 15, n))
    cam = scenes.look_at((0.3, -0.2, -0.5), (0.0, 0.0, 3.0), 40, 32, 36.0, bg=(0.2, 0.1, 0.3))
    return scenes.make_scene("gc-mip", means, ls, q, logits, 3, sh, [cam], dtype=np.float64)


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_with_the_factor_matches_central_differences(seed):
    s = _gc_scene(seed)
    cam = s.cameras[0]
    target = np.random.default_rng(20 + seed).uniform(0, 1, (3, cam.height, cam.width))

    def loss_and_structure():
        r = oracle.Oracle(s, cam, mip_comp=True).render()
        L = oracle.loss(r["image"], target, 0.2, with_grad=False)[0]
        return L, (r["n_contrib"].tobytes(), int(r["stats"][1]))

    o = oracle.Oracle(s, cam, mip_comp=True)
    r = o.render()
    assert 0.05 < r["final_T"].mean() < 0.999  # the splats cover part of the image
    _, _, _, dimg = oracle.loss(r["image"], target, 0.2)
    g = o.backward(dimg)
    h = 1e-6
    checked = skipped = 0
    for name in ("means", "log_scales", "quats", "opacity_logits"):
        arr = getattr(s, name)
        for k in range(arr.size):
            idx = np.unravel_index(k, arr.shape)
            if idx[-1] >= s.n:
                continue
            base = arr[idx]
            arr[idx] = base + h
            Lp, sp = loss_and_structure()
            arr[idx] = base - h
            Lm, sm = loss_and_structure()
            arr[idx] = base
            if sp != sm:
                skipped += 1
                continue
            num = (Lp - Lm) / (2 * h)
            assert abs(num - g[name][idx]) <= 1e-6 * abs(num) + 2e-9, (name, idx, num, g[name][idx])
            checked += 1
    assert checked >= 120 and skipped <= 0.03 * (checked + skipped)
    # the factor moves the log-scale gradient: without it the same scene differs
    g0 = oracle.Oracle(s, cam).backward(dimg)
    assert np.abs(g0["log_scales"] - g["log_scales"]).max() > 1e-3 * np.abs(g["log_scales"]).max()
