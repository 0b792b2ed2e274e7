"""The float64 oracle against the numbers the pages print for worked examples,
closed forms, library routines and invariants (no GPU needed)."""
import math

import numpy as np
import pytest

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes


def screen_row(u, v, A, B, C, o, rgb):
    return [u, v, A, B, C, o, *rgb]


def one_camera(W=64, H=64, f=64.0, bg=(0.0, 0.0, 0.0)):
    return scenes.identity_camera(W, H, f, bg=bg)


def scene_of(means, sigmas, logits, rgbs, cam, quats=None, sh_degree=0, sh_hi=None):
    means = np.asarray(means, np.float64).T
    n = means.shape[1]
    ls = np.log(np.broadcast_to(np.asarray(sigmas, np.float64).reshape(-1, 1)
                                if np.ndim(sigmas) == 1 else np.asarray(sigmas), (n, 3))).T.copy()
    q = np.tile(np.array([[1.0], [0.0], [0.0], [0.0]]), (1, n)) if quats is None else np.asarray(quats).T
    K = (sh_degree + 1) ** 2
    sh = np.zeros((3, K, n))
    sh[:, 0, :] = np.asarray(rgbs, np.float64).T
    if sh_hi is not None:
        sh[:, 1:, :] = sh_hi
    return scenes.make_scene("pin", means, ls, q, np.asarray(logits, np.float64), sh_degree, sh, [cam],
                             dtype=np.float64)


# ------------------------------------------------------------ compositing order
def test_two_gaussian_compositing_screen(gold):
    g = gold("compositing_two_gaussians.txt")
    red = screen_row(0, 0, 1, 0, 1, g["near_opacity"], (1, 0, 0))
    blue = screen_row(0, 0, 1, 0, 1, g["far_opacity"], (0, 0, 1))
    scr = np.array([red, blue])
    rgb, _, _ = oracle.blend_screen(scr, [0, 1], 0.0, 0.0)
    np.testing.assert_allclose(rgb, g["near_first_rgb"], atol=1e-12)
    rgb, _, _ = oracle.blend_screen(scr, [1, 0], 0.0, 0.0)
    np.testing.assert_allclose(rgb, g["far_first_rgb"], atol=1e-12)


def test_two_gaussian_compositing_through_projection_and_sort(gold):
    """Same example through the full path: depth sort must put the near red one first."""
    g = gold("compositing_two_gaussians.txt")
    cam = one_camera()
    # Same projected spread: sigma/depth equal for both.
    zn, zf = g["near_depth"], g["far_depth"]
    logit = lambda o: math.log(o / (1 - o))
    # list the far one first so only the depth sort can restore the order
    s = scene_of([[0, 0, zf], [0, 0, zn]], [0.02 * zf, 0.02 * zn],
                 [logit(g["far_opacity"]), logit(g["near_opacity"])], [(0, 0, 1), (1, 0, 0)], cam)
    o = oracle.Oracle(s, cam)
    img = o.render()["image"]
    np.testing.assert_allclose(img[:, 32, 32], g["near_first_rgb"], atol=1e-12)


# -------------------------------------------------------------- projected spread
def test_projected_spread(gold):
    g = gold("projected_spread.txt")
    cam = one_camera(f=g["focal"])
    for depth, expect in ((g["depth_a"], g["sigma2d_a"]), (g["depth_b"], g["sigma2d_b"])):
        s = scene_of([[0, 0, depth]], [g["sigma_world"]], [0.0], [(1, 1, 1)], cam)
        cov = oracle.Oracle(s, cam).preprocess()["cov2d"][0]
        # the dilated covariance carries the 0.3 px^2 filter on its diagonal
        assert math.sqrt(cov[0] - 0.3) == pytest.approx(expect, rel=1e-12)
        assert math.sqrt(cov[2] - 0.3) == pytest.approx(expect, rel=1e-12)
        assert cov[1] == pytest.approx(0.0, abs=1e-12)


# ------------------------------------------------------------ opacity gradient
def test_opacity_gradient_and_step(gold):
    g = gold("opacity_step.txt")
    op, col, bg, tgt = g["opacity"], g["color"], g["background"], g["target"]
    scr = np.array([screen_row(0, 0, 1, 0, 1, op, col)])
    rgb, _, _ = oracle.blend_screen(scr, [0], 0, 0, bg=bg)
    np.testing.assert_allclose(rgb, g["rendered"], atol=1e-12)
    assert np.sum((rgb - tgt) ** 2) == pytest.approx(g["loss"], abs=1e-12)
    _, _, sg = oracle.blend_screen(scr, [0], 0, 0, bg=bg, dldI=2 * (rgb - tgt))
    assert sg[0, 5] == pytest.approx(g["dloss_dopacity"], abs=1e-12)
    new_op = op - g["learning_rate"] * sg[0, 5]
    assert new_op == pytest.approx(g["opacity_after_step"], abs=1e-12)
    scr2 = np.array([screen_row(0, 0, 1, 0, 1, new_op, col)])
    rgb2, _, _ = oracle.blend_screen(scr2, [0], 0, 0, bg=bg)
    assert np.sum((rgb2 - tgt) ** 2) < g["loss"]


def test_opacity_gradient_through_parameters(gold):
    """The same pixel through preprocess + blend backward: dL/dlogit = dL/do * o (1 - o)."""
    g = gold("opacity_step.txt")
    cam = one_camera(bg=tuple(g["background"]))
    s = scene_of([[0, 0, 5]], [0.1], [0.0], [tuple(g["color"])], cam)
    o = oracle.Oracle(s, cam)
    img = o.render()["image"]
    np.testing.assert_allclose(img[:, 32, 32], g["rendered"], atol=1e-12)
    dimg = np.zeros_like(img)
    dimg[:, 32, 32] = 2 * (img[:, 32, 32] - g["target"])
    gr = o.backward(dimg)
    assert gr["screen"][0, 5] == pytest.approx(g["dloss_dopacity"], abs=1e-12)
    assert gr["opacity_logits"][0] == pytest.approx(g["dloss_dopacity"] * 0.25, abs=1e-12)


# ------------------------------------------------------------- blend weights
def test_blend_weights(gold):
    g = gold("blend_weights.txt")
    a1, a2 = g["alphas"]
    scr = np.array([screen_row(0, 0, 1, 0, 1, a1, (1, 0, 0)),
                    screen_row(0, 0, 1, 0, 1, a2, (0, 1, 0))])
    rgb, T, _ = oracle.blend_screen(scr, [0, 1], 0, 0, bg=(0, 0, 1))
    np.testing.assert_allclose(rgb[:2], g["weights"], atol=1e-12)
    assert rgb[2] == pytest.approx(g["background_weight"], abs=1e-12)
    assert T == pytest.approx(g["background_weight"], abs=1e-12)
    assert rgb.sum() == pytest.approx(1.0, abs=1e-12)


def test_weights_plus_transmittance_is_one():
    """With every colour 1 and a black background, each pixel equals 1 - T."""
    s = scenes.tiny(seed=5)
    s.sh[:, 0, : s.n] = 1.0
    r = oracle.Oracle(s, s.cameras[0]).render()
    for ch in range(3):
        np.testing.assert_allclose(r["image"][ch] + r["final_T"], 1.0, atol=1e-12)
    assert r["stats"][1] > 0


# ------------------------------------------------------ centre gradient example
def test_centre_gradient_example(gold):
    g = gold("centre_gradient.txt")
    d = g["pixel"] - g["centre"]
    inv = 1.0 / g["sigma"] ** 2  # conic of an isotropic unit Gaussian, no dilation
    scr = np.array([screen_row(-d, 0.0, inv, 0.0, inv, g["opacity"], (1, 1, 1))])
    rgb, _, _ = oracle.blend_screen(scr, [0], 0, 0)
    assert rgb[0] == pytest.approx(g["rendered"], abs=5e-8)
    dl = np.array([g["dloss_dI"], 0, 0]) if rgb[0] < g["target"] else np.array([1.0, 0, 0])
    _, _, sg = oracle.blend_screen(scr, [0], 0, 0, dldI=dl)
    # dL/du of the screen centre = dL/dI * dI/dm
    assert sg[0, 0] == pytest.approx(g["dloss_dI"] * g["dI_dm"], abs=5e-8)
    new_centre = g["centre"] - g["step"] * sg[0, 0]
    assert new_centre == pytest.approx(g["centre_after_step"], abs=5e-9)
    scr2 = np.array([screen_row(new_centre - g["pixel"], 0.0, inv, 0.0, inv, g["opacity"], (1, 1, 1))])
    rgb2, _, _ = oracle.blend_screen(scr2, [0], 0, 0)
    assert rgb2[0] == pytest.approx(g["rendered_after_step"], abs=1e-10)
    assert abs(rgb2[0] - g["target"]) == pytest.approx(g["abs_error_after_step"], abs=1e-10)


# ----------------------------------------------------- thresholds on the walk
def test_alpha_cap_and_floor():
    # cap: opacity 1 at the centre blends at most 0.99
    rgb, T, _ = oracle.blend_screen(np.array([screen_row(0, 0, 1, 0, 1, 1.0, (1, 1, 1))]), [0], 0, 0)
    np.testing.assert_allclose(rgb, 0.99, atol=1e-15)
    assert T == pytest.approx(0.01, abs=1e-15)
    # floor: alpha just under 1/255 is skipped, just over is blended
    below = screen_row(0, 0, 1, 0, 1, 1.0 / 255.0 * (1 - 1e-9), (1, 1, 1))
    above = screen_row(0, 0, 1, 0, 1, 1.0 / 255.0 * (1 + 1e-9), (1, 1, 1))
    rgb, T, _ = oracle.blend_screen(np.array([below]), [0], 0, 0)
    assert rgb[0] == 0.0 and T == 1.0
    rgb, T, _ = oracle.blend_screen(np.array([above]), [0], 0, 0)
    assert rgb[0] > 0.0 and T < 1.0


def test_early_termination_includes_the_crossing_gaussian():
    """Three capped red layers drive T to 1e-6: the third is blended, the green
    fourth one is never reached."""
    reds = [screen_row(0, 0, 1, 0, 1, 1.0, (1, 0, 0)) for _ in range(3)]
    green = screen_row(0, 0, 1, 0, 1, 0.9, (0, 1, 0))
    rgb, T, _ = oracle.blend_screen(np.array(reds + [green]), [0, 1, 2, 3], 0, 0)
    assert rgb[1] == 0.0
    assert T == pytest.approx(1e-6, rel=1e-9)
    assert rgb[0] == pytest.approx(1 - 1e-6, abs=1e-12)


# --------------------------------------------------------------------- loss
def test_loss_combiner_example(gold):
    g = gold("loss_combiner.txt")
    lam = g["lambda"]
    assert (1 - lam) * g["l1"] + lam * (1 - g["ssim"]) == pytest.approx(g["loss"], abs=1e-15)
    rng = np.random.default_rng(0)
    x = rng.uniform(0, 1, (3, 20, 23))
    y = rng.uniform(0, 1, (3, 20, 23))
    L, l1, ssim, _ = oracle.loss(x, y, lam)
    assert L == pytest.approx((1 - lam) * l1 + lam * (1 - ssim), abs=1e-15)
    # lambda = 0 and 1 isolate the two terms
    assert oracle.loss(x, y, 0.0)[0] == pytest.approx(l1, abs=1e-15)
    assert oracle.loss(x, y, 1.0)[0] == pytest.approx(1 - ssim, abs=1e-15)


def test_l1_is_the_mean_absolute_error():
    rng = np.random.default_rng(1)
    x = rng.uniform(0, 1, (3, 17, 9))
    y = rng.uniform(0, 1, (3, 17, 9))
    assert oracle.loss(x, y)[1] == pytest.approx(np.mean(np.abs(x - y)), rel=1e-14)


def _window():
    g = np.exp(-(np.arange(-5, 6) ** 2) / (2 * 1.5 ** 2))
    g /= g.sum()
    return np.outer(g, g)


def test_ssim_matches_library_convolution():
    """SSIM via scipy.ndimage.correlate with zero padding ('constant', cval 0)."""
    from scipy import ndimage
    rng = np.random.default_rng(2)
    x = rng.uniform(0, 1, (3, 24, 31))
    y = np.clip(x + rng.normal(0, 0.2, x.shape), 0, 1)
    w = _window()
    C1, C2 = 0.01 ** 2, 0.03 ** 2
    vals = []
    for c in range(3):
        f = lambda a: ndimage.correlate(a, w, mode="constant", cval=0.0)
        mx, my = f(x[c]), f(y[c])
        sxx = f(x[c] * x[c]) - mx * mx
        syy = f(y[c] * y[c]) - my * my
        sxy = f(x[c] * y[c]) - mx * my
        vals.append(((2 * mx * my + C1) * (2 * sxy + C2)) /
                    ((mx * mx + my * my + C1) * (sxx + syy + C2)))
    assert oracle.loss(x, y)[2] == pytest.approx(np.mean(vals), rel=1e-12)


def test_ssim_closed_forms():
    rng = np.random.default_rng(3)
    x = rng.uniform(0, 1, (3, 15, 15))
    L, l1, ssim, d = oracle.loss(x, x)
    assert ssim == pytest.approx(1.0, abs=1e-13)
    assert L == pytest.approx(0.0, abs=1e-13)
    # the optimum: zero L1 subgradient at zero residual and a stationary SSIM
    np.testing.assert_allclose(d, 0.0, atol=1e-14)
    # constant images a and b on a 40x40 image: in the interior (at least 5 px from
    # every border, where the window lies inside the image) the map is
    # (2ab + C1) / (a^2 + b^2 + C1); the border ring is checked by the library test.
    a, b = 0.3, 0.7
    C1 = 0.01 ** 2
    H = W = 40
    xa = np.full((3, H, W), a)
    yb = np.full((3, H, W), b)
    s_all = oracle.loss(xa, yb)[2] * H * W
    # remove the border ring using the library computation of the same map
    from scipy import ndimage
    w = _window()
    f = lambda m: ndimage.correlate(m, w, mode="constant", cval=0.0)
    ones = np.ones((H, W))
    Wq = f(ones)
    C2 = 0.03 ** 2
    ring = np.ones((H, W), bool)
    ring[5:-5, 5:-5] = False
    mx, my = a * Wq, b * Wq
    sxx = a * a * Wq - mx * mx
    syy = b * b * Wq - my * my
    sxy = a * b * Wq - mx * my
    smap = ((2 * mx * my + C1) * (2 * sxy + C2)) / ((mx * mx + my * my + C1) * (sxx + syy + C2))
    interior = (s_all - smap[ring].sum()) / (~ring).sum()
    assert interior == pytest.approx((2 * a * b + C1) / (a * a + b * b + C1), rel=1e-12)


def test_loss_gradient_central_differences():
    rng = np.random.default_rng(4)
    x = rng.uniform(0, 1, (3, 13, 17))
    y = rng.uniform(0, 1, (3, 13, 17))
    _, _, _, d = oracle.loss(x, y)
    h = 1e-6
    idx = [(c, i, j) for c in range(3) for i in range(13) for j in range(17)]
    for (c, i, j) in idx[::7]:
        xp = x.copy(); xp[c, i, j] += h
        xm = x.copy(); xm[c, i, j] -= h
        num = (oracle.loss(xp, y, with_grad=False)[0] - oracle.loss(xm, y, with_grad=False)[0]) / (2 * h)
        assert d[c, i, j] == pytest.approx(num, rel=1e-6, abs=1e-11)


# --------------------------------------------------------------------- Adam
def test_adam_constant_gradient_closed_form():
    """With a constant gradient the bias-corrected moments are m_hat = g and
    v_hat = g^2 at every step, so each step moves p by lr g / (|g| + eps)."""
    rng = np.random.default_rng(5)
    g0 = rng.normal(0, 1e-2, 100)
    p = rng.normal(0, 1, 100)
    m = np.zeros(100)
    v = np.zeros(100)
    lr, eps = 1e-3, 1e-8
    p_exp = p.copy()
    for t in range(1, 4):
        p, g, m, v = oracle.adam(p, g0, m, v, lr, t, eps=eps)
        p_exp = p_exp - lr * g0 / (np.abs(g0) + eps)
        np.testing.assert_allclose(p, p_exp, rtol=0, atol=1e-15)
        assert not g.any()


def _adam_closed_form(p0, grads, lr, beta1, beta2, eps):
    """Adam's trajectory from the sums the recursion unrolls to (no recursion):
    m_t = (1 - b1) sum_k b1^(t-k) g_k and v_t = (1 - b2) sum_k b2^(t-k) g_k^2,
    divided by the bias corrections 1 - b1^t and 1 - b2^t, then
    p_t = p_(t-1) - lr m_hat_t / (sqrt(v_hat_t) + eps). Returns every p_t, m_t, v_t."""
    p = np.array(p0, np.float64)
    out = []
    for t in range(1, len(grads) + 1):
        m_t = (1 - beta1) * sum(beta1 ** (t - k) * grads[k - 1] for k in range(1, t + 1))
        v_t = (1 - beta2) * sum(beta2 ** (t - k) * grads[k - 1] ** 2 for k in range(1, t + 1))
        m_hat = m_t / (1 - beta1 ** t)
        v_hat = v_t / (1 - beta2 ** t)
        p = p - lr * m_hat / (np.sqrt(v_hat) + eps)
        out.append((p.copy(), m_t, v_t))
    return out


def test_adam_varying_gradients_match_the_unrolled_sums():
    """Three steps with different gradients (signs and sizes change from step to
    step) and beta1 != beta2: the oracle's recursion must give the unrolled
    moment sums, their bias corrections at the step's own power, and the
    parameter trajectory. The constant-gradient test cannot tell beta1 from
    beta2 (m_hat = g, v_hat = g^2 whichever decays which); this one can."""
    rng = np.random.default_rng(15)
    n = 64
    p0 = rng.normal(0, 1, n)
    grads = [rng.normal(0, 1, n) * s for s in (1.0, 3e-2, 5.0)]
    grads[1][::3] *= -40.0  # some gradients flip sign and grow between steps
    lr, b1, b2, eps = 1e-2, 0.9, 0.999, 1e-8
    want = _adam_closed_form(p0, grads, lr, b1, b2, eps)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t, g in enumerate(grads, start=1):
        p, gz, m, v = oracle.adam(p, g, m, v, lr, t, beta1=b1, beta2=b2, eps=eps)
        wp, wm, wv = want[t - 1]
        np.testing.assert_allclose(m, wm, rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(v, wv, rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(p, wp, rtol=1e-13, atol=1e-15)
        assert not gz.any()
    # The same sums with the betas swapped, or with a bias correction one power
    # off, land far outside that tolerance: the comparison above can see both.
    swapped = _adam_closed_form(p0, grads, lr, b2, b1, eps)[-1][0]
    assert np.abs(swapped - p).max() > 1e-4
    off_by_one = p0.copy()
    for t in range(1, 4):
        m_t = (1 - b1) * sum(b1 ** (t - k) * grads[k - 1] for k in range(1, t + 1))
        v_t = (1 - b2) * sum(b2 ** (t - k) * grads[k - 1] ** 2 for k in range(1, t + 1))
        off_by_one = off_by_one - lr * (m_t / (1 - b1 ** (t + 1))) / (np.sqrt(v_t / (1 - b2 ** t)) + eps)
    assert np.abs(off_by_one - p).max() > 1e-4


def test_adam_scalar_worked_by_hand():
    """Two steps on one scalar, every intermediate written out by hand:
    g1 = 2:  m1 = 0.2,  v1 = 0.004,  m_hat = 2,  v_hat = 4,  p1 = 1 - 0.1 * 2 / (2 + eps)
    g2 = -1: m2 = 0.9 * 0.2 - 0.1 = 0.08,  v2 = 0.999 * 0.004 + 0.001 = 0.004996,
             m_hat = 0.08 / 0.19,  v_hat = 0.004996 / 0.001999,
             p2 = p1 - 0.1 * m_hat / (sqrt(v_hat) + eps)."""
    eps = 1e-8
    p, _, m, v = oracle.adam([1.0], [2.0], [0.0], [0.0], 0.1, 1, eps=eps)
    assert m[0] == pytest.approx(0.2, rel=1e-15)
    assert v[0] == pytest.approx(0.004, rel=1e-14)
    p1 = 1.0 - 0.1 * 2.0 / (2.0 + eps)
    assert p[0] == pytest.approx(p1, rel=1e-15)
    p, _, m, v = oracle.adam(p, [-1.0], m, v, 0.1, 2, eps=eps)
    assert m[0] == pytest.approx(0.08, rel=1e-14)
    assert v[0] == pytest.approx(0.004996, rel=1e-14)
    m_hat = 0.08 / 0.19
    v_hat = 0.004996 / 0.001999
    assert p[0] == pytest.approx(p1 - 0.1 * m_hat / (math.sqrt(v_hat) + eps), rel=1e-14)


def test_adam_matches_torch_float64():
    """Library pin: torch.optim.Adam in float64 (its default betas and eps are the
    oracle's) over four steps of changing gradients, per-group learning rates."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(16)
    n = 40
    p0 = rng.normal(0, 1, n)
    grads = [rng.normal(0, 1, n) * (10.0 ** rng.uniform(-3, 1)) for _ in range(4)]
    for lr in (1e-3, 0.05):
        w = torch.tensor(p0.copy(), dtype=torch.float64, requires_grad=True)
        opt = torch.optim.Adam([w], lr=lr, betas=(0.9, 0.999), eps=1e-8)
        p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
        for t, g in enumerate(grads, start=1):
            w.grad = torch.tensor(g, dtype=torch.float64)
            opt.step()
            p, _, m, v = oracle.adam(p, g, m, v, lr, t)
            np.testing.assert_allclose(p, w.detach().numpy(), rtol=1e-12, atol=1e-15)
            st = opt.state[w]
            np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-13, atol=1e-300)
            np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-13, atol=1e-300)


# ------------------------------------------------------------------------ SH
def test_sh_printed_constants(gold):
    g = gold("sh_constants.txt")
    rng = np.random.default_rng(6)
    dirs = rng.normal(size=(50, 3))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    Y = oracle.sh_basis(3, dirs)
    x, y, z = dirs.T
    poly = {"x": x, "y": y, "z": z, "xy": x * y, "yz": y * z, "xz": x * z,
            "2zz-xx-yy": 2 * z * z - x * x - y * y, "xx-yy": x * x - y * y}
    for k in range(1, 9):
        const, p = g[f"Y{k}"].split()
        # printed to 7 decimals
        np.testing.assert_allclose(Y[:, k], float(const) * poly[p], atol=6e-8)
    np.testing.assert_allclose(Y[:, 0], 1.0)


def test_sh_orthonormal_by_quadrature():
    """Gauss-Legendre in cos(theta) x uniform in phi integrates products of
    degree <= 6 exactly: the real SH (k >= 1) are orthonormal and orthogonal to 1."""
    nz, nphi = 12, 16
    zs, wz = np.polynomial.legendre.leggauss(nz)
    phis = 2 * np.pi * np.arange(nphi) / nphi
    Z, PHI = np.meshgrid(zs, phis, indexing="ij")
    Wt = np.repeat(wz[:, None], nphi, axis=1) * (2 * np.pi / nphi)
    st = np.sqrt(1 - Z ** 2)
    dirs = np.stack([st * np.cos(PHI), st * np.sin(PHI), Z], -1).reshape(-1, 3)
    Y = oracle.sh_basis(3, dirs)
    G = (Y * Wt.reshape(-1, 1)).T @ Y
    np.testing.assert_allclose(G[1:, 1:], np.eye(15), atol=1e-12)
    np.testing.assert_allclose(G[0, 1:], 0.0, atol=1e-12)
    assert G[0, 0] == pytest.approx(4 * np.pi, rel=1e-12)


def test_sh_degree_zero_is_the_base_colour():
    s = scenes.small()
    o = oracle.Oracle(s, s.cameras[0], active_degree=0)
    pp = o.preprocess()
    vis = pp["touched"] > 0
    base = np.maximum(s.sh[:, 0, : s.n].T.astype(np.float64), 0.0)
    np.testing.assert_allclose(pp["screen"][vis, 6:9], base[vis], atol=0)


# --------------------------------------------------------- rotation, covariance
def test_rotation_and_covariance_match_library():
    from scipy.spatial.transform import Rotation
    rng = np.random.default_rng(7)
    for _ in range(20):
        q = rng.normal(size=4) * rng.uniform(0.2, 3.0)
        ls = rng.normal(-2, 0.7, 3)
        R, S = oracle.rotation_cov(q, ls)
        Rl = Rotation.from_quat([q[1], q[2], q[3], q[0]]).as_matrix()  # scalar-last
        np.testing.assert_allclose(R, Rl, atol=1e-13)
        s2 = np.exp(2 * ls)
        np.testing.assert_allclose(np.sort(np.linalg.eigvalsh(S)), np.sort(s2), rtol=1e-10)
        for i in range(3):
            np.testing.assert_allclose(S @ Rl[:, i], s2[i] * Rl[:, i], atol=1e-12)


def test_projection_matches_sampled_pinhole():
    """EWA: the screen covariance minus the 0.3 px^2 filter is the covariance of
    exactly projected samples, to first order in sigma/Z (J and W pinned by sampling)."""
    rng = np.random.default_rng(8)
    cam = scenes.look_at((1.0, -0.5, -6.0), (0.2, 0.1, 0.0), 128, 96, 150.0)
    mean = np.array([0.6, -0.3, 0.4])
    q = rng.normal(size=4)
    ls = np.log([0.004, 0.009, 0.002])
    s = scenes.make_scene("mc", mean.reshape(3, 1), ls.reshape(3, 1), q.reshape(4, 1),
                          np.array([0.0]), 0, np.ones((3, 1, 1)), [cam], dtype=np.float64)
    pp = oracle.Oracle(s, cam).preprocess()
    _, Sig = oracle.rotation_cov(q, ls)
    pts = rng.multivariate_normal(mean, Sig, 400_000)
    R = cam.R.astype(np.float64)
    pc = pts @ R.T + cam.t.astype(np.float64)
    uv = np.stack([cam.fx * pc[:, 0] / pc[:, 2] + cam.cx, cam.fy * pc[:, 1] / pc[:, 2] + cam.cy], 1)
    emp = np.cov(uv.T)
    a, b, c = pp["cov2d"][0]
    model = np.array([[a - 0.3, b], [b, c - 0.3]])
    np.testing.assert_allclose(model, emp, rtol=0.02, atol=0.02 * np.abs(emp).max())
    pc0 = R @ mean + cam.t
    u0 = cam.fx * pc0[0] / pc0[2] + cam.cx
    v0 = cam.fy * pc0[1] / pc0[2] + cam.cy
    np.testing.assert_allclose(pp["screen"][0, :2], [u0, v0], rtol=1e-12)
    assert pp["depth"][0] == pytest.approx(pc0[2], rel=1e-14)


def test_conic_is_the_inverse_covariance_and_radius_from_eigenvalue():
    s = scenes.small()
    pp = oracle.Oracle(s, s.cameras[0]).preprocess()
    vis = np.nonzero(pp["touched"] > 0)[0][:500]
    for i in vis:
        a, b, c = pp["cov2d"][i]
        A, B, C = pp["screen"][i, 2:5]
        np.testing.assert_allclose(np.array([[A, B], [B, C]]) @ np.array([[a, b], [b, c]]),
                                   np.eye(2), atol=1e-9)
        lmax = np.linalg.eigvalsh(np.array([[a, b], [b, c]]))[-1]
        assert pp["radius"][i] == pytest.approx(3 * math.sqrt(lmax), rel=1e-9)
