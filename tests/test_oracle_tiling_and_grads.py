"""The oracle's tile lists against brute force, and its whole backward (blend,
projection, SH view-direction path, loss) against float64 central differences
of its own forward, as the taosengine page's "Proving the blame is right" section
prescribes."""
import math

import numpy as np
import pytest

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes


def test_rect_is_every_tile_meeting_the_radius_box():
    s = scenes.small()
    cam = s.cameras[0]
    o = oracle.Oracle(s, cam)
    pp = o.preprocess()
    tx, ty = o.tiles
    for i in np.nonzero(pp["touched"] > 0)[0][:300]:
        u, v = pp["screen"][i, :2]
        r = pp["radius"][i]
        xs = [t for t in range(tx) if 16 * t <= u + r and 16 * t + 15 >= u - r]
        ys = [t for t in range(ty) if 16 * t <= v + r and 16 * t + 15 >= v - r]
        x0, y0, x1, y1 = pp["rect"][i]
        assert (x0, x1) == (xs[0], xs[-1]) and (y0, y1) == (ys[0], ys[-1])
        assert pp["touched"][i] == len(xs) * len(ys)


def test_sorted_lists_match_brute_force_per_tile():
    s = scenes.small()
    o = oracle.Oracle(s, s.cameras[0])
    pp = o.preprocess()
    srt = o.sorted()
    tx, ty = o.tiles
    rect = pp["rect"]
    keys = pp["depth_key"].view(np.uint32)
    assert srt["ids"].size == pp["touched"].sum()
    for t in range(tx * ty):
        x, y = t % tx, t // tx
        inside = np.nonzero((pp["touched"] > 0) & (rect[:, 0] <= x) & (x <= rect[:, 2]) &
                            (rect[:, 1] <= y) & (y <= rect[:, 3]))[0]
        order = inside[np.lexsort((inside, keys[inside]))]  # depth bits, then id
        lo, hi = srt["ranges"][t]
        if order.size == 0:
            assert lo == hi
        np.testing.assert_array_equal(srt["ids"][lo:hi], order)
        assert (srt["tiles"][lo:hi] == t).all()


def test_tiled_render_equals_per_pixel_brute_force():
    """Each pixel blended over every Gaussian whose rect covers its tile, ordered by
    (depth, id) with a library sort, equals the tiled render bit for bit."""
    s = scenes.tiny()
    cam = s.cameras[0]
    o = oracle.Oracle(s, cam)
    pp = o.preprocess()
    r = o.render()
    keys = pp["depth_key"].view(np.uint32)
    for py in range(0, 64, 3):
        for px in range(0, 64, 5):
            x, y = px // 16, py // 16
            rect = pp["rect"]
            cand = np.nonzero((pp["touched"] > 0) & (rect[:, 0] <= x) & (x <= rect[:, 2]) &
                              (rect[:, 1] <= y) & (y <= rect[:, 3]))[0]
            order = cand[np.lexsort((cand, keys[cand]))]
            rgb, T, _ = oracle.blend_screen(pp["screen"], order, px, py, bg=cam.bg)
            np.testing.assert_array_equal(rgb, r["image"][:, py, px])
            assert T == r["final_T"][py, px]


def _gradcheck_scene(seed=0, n=12, W=40, H=32, sh_degree=3):
    rng = np.random.default_rng(seed)
    means = np.stack([rng.uniform(-0.6, 0.6, n), rng.uniform(-0.45, 0.45, n), rng.uniform(2.0, 4.0, n)])
    ls = rng.normal(math.log(0.12), 0.3, (3, n))
    q = rng.normal(size=(4, n))
    logits = rng.normal(0.0, 1.0, n)
    K = (sh_degree + 1) ** 2
    sh = np.zeros((3, K, n))
    sh[:, 0] = rng.uniform(0.3, 1.0, (3, n))
    sh[:, 1:] = rng.normal(0.0, 0.3, (3, K - 1, n))
    cam = scenes.look_at((0.3, -0.2, -0.5), (0.0, 0.0, 3.0), W, H, 36.0, bg=(0.2, 0.1, 0.3))
    return scenes.make_scene("gc", means, ls, q, logits, sh_degree, sh, [cam], dtype=np.float64)


def _loss_and_structure(scene, cam, target):
    o = oracle.Oracle(scene, cam)
    r = o.render()
    L = oracle.loss(r["image"], target, 0.2, with_grad=False)[0]
    return L, (r["n_contrib"].tobytes(), int(r["stats"][1]), int(r["ambiguous"].sum()))


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_central_differences(seed):
    s = _gradcheck_scene(seed)
    cam = s.cameras[0]
    target = np.random.default_rng(10 + seed).uniform(0, 1, (3, cam.height, cam.width))
    o = oracle.Oracle(s, cam)
    r = o.render()
    _, _, _, dimg = oracle.loss(r["image"], target, 0.2)
    g = o.backward(dimg)
    h = 1e-6
    checked = skipped = 0
    worst = 0.0
    for name in scenes.GROUP_NAMES:
        arr = getattr(s, name)
        grad = g[name]
        flat_idx = [np.unravel_index(k, arr.shape) for k in range(arr.size)
                    if np.unravel_index(k, arr.shape)[-1] < s.n]
        for idx in flat_idx:
            base = arr[idx]
            arr[idx] = base + h
            Lp, sp = _loss_and_structure(s, cam, target)
            arr[idx] = base - h
            Lm, sm = _loss_and_structure(s, cam, target)
            arr[idx] = base
            if sp != sm:  # a threshold decision flipped inside +-h: not differentiable there
                skipped += 1
                continue
            num = (Lp - Lm) / (2 * h)
            err = abs(num - grad[idx])
            worst = max(worst, err / (abs(num) + 1e-7))
            assert err <= 1e-6 * abs(num) + 2e-9, (name, idx, num, grad[idx])
            checked += 1
    assert skipped <= 0.02 * (checked + skipped)
    assert checked > 600


def test_view_direction_path_is_included():
    """Zeroing the SH higher bands must change the position gradient: the colour
    depends on the view direction and so on the mean."""
    s = _gradcheck_scene(3)
    cam = s.cameras[0]
    target = np.random.default_rng(4).uniform(0, 1, (3, cam.height, cam.width))
    o = oracle.Oracle(s, cam)
    _, _, _, dimg = oracle.loss(o.render()["image"], target, 0.2)
    g_full = o.backward(dimg)["means"]
    s0 = s.copy()
    s0.sh[:, 1:, :] = 0.0
    o0 = oracle.Oracle(s0, cam)
    _, _, _, dimg0 = oracle.loss(o0.render()["image"], target, 0.2)
    g0 = o0.backward(dimg0)["means"]
    assert np.abs(g_full - g0).max() > 1e-4


def test_split_backward_equals_whole_backward():
    """The blend backward over two row bands plus the projection backward over
    two Gaussian slices reproduce the one-call backward exactly (the parts are
    sums over disjoint pixels and maps over disjoint Gaussians)."""
    s = scenes.tiny()
    cam = s.cameras[0]
    o = oracle.Oracle(s, cam)
    rng = np.random.default_rng(3)
    dimage = rng.normal(size=(3, cam.height, cam.width))
    whole = o.backward(dimage)
    sg = np.zeros((s.n, 9))
    mid = cam.height // 2
    o.blend_backward_rows(0, mid, dimage, sg)
    o.blend_backward_rows(mid, cam.height, dimage, sg)
    np.testing.assert_allclose(sg, whole["screen"], rtol=1e-12, atol=1e-15)
    parts = {k: np.full_like(v, np.nan) for k, v in whole.items() if k != "screen"}
    o.project_backward(sg, 0, s.n // 3, parts)
    o.project_backward(sg, s.n // 3, s.n, parts)
    for k, v in parts.items():
        idx = (Ellipsis, slice(0, s.n))
        np.testing.assert_allclose(v[idx], whole[k][idx], rtol=1e-12, atol=1e-15, err_msg=k)


def test_opacity_aware_rect_drops_only_tiles_without_contribution():
    """The opacity-aware tile rect (falloff cut min(4.5, ln(255 o)) instead of
    4.5) keeps a subset of the 3-sigma rect, drops only tiles in which the
    Gaussian's alpha stays below 1/255 at every pixel (checked by brute force),
    and leaves the rendered image and transmittance unchanged."""
    s = scenes.small()
    cam = s.cameras[0]
    o3 = oracle.Oracle(s, cam)
    oa = oracle.Oracle(s, cam, opacity_rect=True)
    p3, pa = o3.preprocess(), oa.preprocess()
    assert pa["touched"].sum() < p3["touched"].sum()
    vis = pa["touched"] > 0
    assert np.all(p3["touched"][vis] > 0)
    r3, ra = p3["rect"], pa["rect"]  # x0, y0, x1, y1
    assert np.all(ra[vis, 0] >= r3[vis, 0]) and np.all(ra[vis, 1] >= r3[vis, 1])
    assert np.all(ra[vis, 2] <= r3[vis, 2]) and np.all(ra[vis, 3] <= r3[vis, 3])
    # every pixel of a dropped tile is below the alpha floor
    changed = np.nonzero(p3["touched"] != pa["touched"])[0]
    assert changed.size > 100
    tx_n, ty_n = o3.tiles
    for i in changed[:400]:
        u, v, A, B, C, o = p3["screen"][i, :6]
        x0, y0, x1, y1 = r3[i]
        keep = np.zeros((ty_n, tx_n), bool)
        if pa["touched"][i] > 0:
            keep[ra[i, 1]:ra[i, 3] + 1, ra[i, 0]:ra[i, 2] + 1] = True
        for ty in range(y0, y1 + 1):
            for tx in range(x0, x1 + 1):
                if keep[ty, tx]:
                    continue
                ys, xs = np.mgrid[16 * ty:16 * ty + 16, 16 * tx:16 * tx + 16]
                dx, dy = xs - u, ys - v
                alpha = o * np.exp(-(0.5 * A * dx * dx + B * dx * dy + 0.5 * C * dy * dy))
                assert alpha.max() < 1.0 / 255.0, (i, tx, ty, alpha.max())
    i3, ia = o3.render(), oa.render()
    np.testing.assert_allclose(ia["image"], i3["image"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ia["final_T"], i3["final_T"], rtol=0, atol=1e-12)


def test_replay_without_flips_is_the_plain_walk_and_flips_change_only_ambiguous_pixels():
    """The replay walk (test support for decisions a float32 renderer may take
    either way) with no flip is the plain walk bit for bit; flipping changes
    nothing at a pixel without near-threshold decisions, and at a pixel with
    one it gives the walk with that decision taken the other way."""
    s = scenes.small()
    cam = s.cameras[0]
    o = oracle.Oracle(s, cam)
    ys, xs = np.mgrid[0:cam.height, 0:cam.width]
    px, py = xs.ravel(), ys.ravel()
    plain = o.render_pixels(px, py)
    rep = o.replay_pixels(px, py, 0)
    np.testing.assert_array_equal(rep["rgb"], plain["rgb"])
    np.testing.assert_array_equal(rep["T"], plain["T"])
    np.testing.assert_array_equal(rep["n_contrib"], plain["n_contrib"])
    amb = plain["ambiguous"].astype(bool)
    np.testing.assert_array_equal(rep["n_amb"] > 0, amb)
    assert 0 < amb.sum() < 0.02 * amb.size
    flipped = o.replay_pixels(px, py, 0xffffffff)
    np.testing.assert_array_equal(flipped["rgb"][~amb], plain["rgb"][~amb])
    changed = np.any(flipped["rgb"][amb] != plain["rgb"][amb], axis=1)
    assert changed.mean() > 0.9
    # a flipped alpha decision moves the pixel by about one contribution at the floor
    d = np.abs(flipped["rgb"][amb] - plain["rgb"][amb]).max(axis=1)
    assert np.median(d) < 1e-2
