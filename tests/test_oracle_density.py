"""The oracle's adaptive density control against what the pages fix
(study notes, "Where to add capacity" / "A separate heuristic": average
screen-gradient magnitude over the views that saw a Gaussian, small ones
cloned and large ones split, very low opacity pruned, reset to opacity at
most 0.01; "Densification": split halves shrink by 1.6, new Gaussians restart
their moments) and what the mathematics fixes (split children are draws from
the parent's own Gaussian N(mean, R S^2 R^T))."""
import math

import numpy as np

import oracle


def _set(n):
    rng = np.random.default_rng(4)
    p = dict(means=rng.normal(size=(3, n)), log_scales=np.full((3, n), math.log(0.01)),
             quats=rng.normal(size=(4, n)), opacity_logits=np.zeros(n),
             sh=rng.uniform(size=(3, 16, n)))
    m = {k: rng.normal(size=v.shape) for k, v in p.items()}
    v = {k: rng.uniform(size=val.shape) for k, val in p.items()}
    return p, m, v


def test_densify_categories_and_order():
    p, m, v = _set(6)
    p["opacity_logits"][0] = -6.0          # opacity 0.0025 < 0.005: pruned
    p["log_scales"][:, 2] = math.log(0.5)  # large
    p["log_scales"][1, 5] = math.log(0.5)
    p["opacity_logits"][5] = -8.0          # large and flagged, but pruned first
    accum = np.array([9.0, 3.0, 4.0, 0.1, 50.0, 9.0])
    count = np.array([1, 2, 2, 1, 0, 1])   # averages 9, 1.5, 2, 0.1, unseen, 9
    normals = np.random.default_rng(1).normal(size=(6, 2, 3))
    out_p, out_m, out_v, n_out = oracle.densify(p, m, v, 6, accum, count, normals, grad_threshold=1.0,
                                                scale_threshold=0.1, min_opacity=0.005)
    # kept 1, 3, 4; clone of 1; two children of 2
    assert n_out == 6
    for g in p:
        for col, i in enumerate((1, 3, 4, 1)):
            np.testing.assert_array_equal(out_p[g][..., col], p[g][..., i])
        for col, i in enumerate((1, 3, 4)):
            np.testing.assert_array_equal(out_m[g][..., col], m[g][..., i])
            np.testing.assert_array_equal(out_v[g][..., col], v[g][..., i])
        assert not out_m[g][..., 3:].any() and not out_v[g][..., 3:].any()
    for col in (4, 5):
        np.testing.assert_allclose(np.exp(out_p["log_scales"][:, col]), np.exp(p["log_scales"][:, 2]) / 1.6)
        for g in ("quats", "opacity_logits", "sh"):
            np.testing.assert_array_equal(out_p[g][..., col], p[g][..., 2])
    assert not np.allclose(out_p["means"][:, 4], out_p["means"][:, 5])


def test_split_children_follow_the_parents_gaussian():
    """The children's offsets from the parent's mean have the parent's
    covariance R diag(s^2) R^T, computed by the oracle's separate covariance
    routine (Monte Carlo, 40 000 children)."""
    n = 20000
    q = np.array([0.8, 0.3, -0.4, 0.35])
    ls = np.log(np.array([0.6, 0.15, 0.3]))
    p = dict(means=np.tile(np.array([[0.5], [-1.0], [2.0]]), n), log_scales=np.tile(ls[:, None], n),
             quats=np.tile(q[:, None], n), opacity_logits=np.ones(n), sh=np.zeros((3, 1, n)))
    zeros = {k: np.zeros_like(val) for k, val in p.items()}
    normals = np.random.default_rng(7).normal(size=(n, 2, 3))
    out_p, _, _, n_out = oracle.densify(p, zeros, zeros, n, np.full(n, 5.0), np.ones(n), normals,
                                        grad_threshold=1.0, scale_threshold=0.1, min_opacity=0.01)
    assert n_out == 2 * n
    d = out_p["means"] - np.array([[0.5], [-1.0], [2.0]])
    _, Sigma = oracle.rotation_cov(q, ls)
    emp = d @ d.T / d.shape[1]
    assert np.abs(emp - Sigma).max() < 0.02 * np.abs(Sigma).max()


def test_opacity_reset_clamps_to_the_cap():
    logits = np.array([3.0, 0.0, -4.0, -10.0])
    out, m, v = oracle.opacity_reset(logits, np.ones(4), np.ones(4), 0.01)
    o = 1.0 / (1.0 + np.exp(-out))
    assert np.all(o <= 0.01 + 1e-15)
    np.testing.assert_allclose(o[:3], 0.01, rtol=1e-12)
    assert out[3] == -10.0  # already below: unchanged
    assert not m.any() and not v.any()


def test_stats_are_the_norm_of_the_centre_gradient_of_seen_gaussians():
    sg = np.zeros((3, 9))
    sg[0, :2] = (3.0, 4.0)
    sg[1, :2] = (1.0, 0.0)
    sg[2, :2] = (2.0, 2.0)
    norm, cnt = oracle.densify_stats(sg, np.array([2, 0, 1]))
    np.testing.assert_allclose(norm, [5.0, 0.0, math.sqrt(8.0)])
    np.testing.assert_array_equal(cnt, [1, 0, 1])
