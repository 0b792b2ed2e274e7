"""The oracle's recycling of dead Gaussians ("How a computer rebuilds a real
place ... Gaussian Splats", section "Densification: cloning the busy blobs,
recycling the dead") against what the section fixes:

* dead (opacity < 0.02) and donors (opacity > 0.4), the largest donors first;
  a worked 6-Gaussian case whose pairing is read off by hand;
* with a zero offset draw the recycled slot is the donor itself, both halves
  shrunk by exactly 1.6;
* the recycled Gaussian is placed from the donor's own Gaussian: over many
  draws its offsets have the donor's covariance R S^2 R^T, built here with
  scipy's rotation (a library routine, not the oracle's);
* slots outside the pairs, and the count, do not change; reshaped Gaussians
  restart their Adam moments.
"""
import math

import numpy as np
import pytest

import oracle

GROUPS = ("means", "log_scales", "quats", "opacity_logits", "sh")


def _logit(o):
    return math.log(o / (1.0 - o))


def _scene(opacities, max_log_scales, seed=0, K=4):
    rng = np.random.default_rng(seed)
    n = len(opacities)
    ls = np.stack([np.asarray(max_log_scales) - d for d in (0.0, 0.3, 0.7)])
    p = dict(means=rng.normal(size=(3, n)), log_scales=ls, quats=rng.normal(size=(4, n)),
             opacity_logits=np.array([_logit(o) for o in opacities]), sh=rng.normal(size=(3, K, n)))
    m = {g: rng.normal(size=p[g].shape) for g in GROUPS}
    v = {g: rng.uniform(0, 1, size=p[g].shape) for g in GROUPS}
    return p, m, v


def test_worked_case_pairs_the_dead_with_the_largest_donors():
    # dead: 0, 4; donors by size: 3 (-1), 1 (-2), 5 (-3); 2 is neither
    p, m, v = _scene([0.01, 0.5, 0.3, 0.9, 0.015, 0.6], [-2.5, -2.0, -0.5, -1.0, -4.0, -3.0])
    z = np.array([[0.3, -0.2, 0.1], [1.0, 0.5, -0.4]])
    P, M, V, pairs = oracle.relocate(p, m, v, 6, z)
    assert pairs == [(0, 3), (4, 1)]
    for i in (2, 5):  # untouched
        for g in GROUPS:
            np.testing.assert_array_equal(P[g][..., i], p[g][..., i])
            np.testing.assert_array_equal(M[g][..., i], m[g][..., i])
            np.testing.assert_array_equal(V[g][..., i], v[g][..., i])
    for i in (0, 1, 3, 4):  # reshaped: moments restart
        for g in GROUPS:
            assert not M[g][..., i].any() and not V[g][..., i].any()
    for d, b in pairs:
        for g in ("quats", "opacity_logits", "sh"):
            np.testing.assert_array_equal(P[g][..., d], p[g][..., b])
            np.testing.assert_array_equal(P[g][..., b], p[g][..., b])
        np.testing.assert_array_equal(P["means"][:, b], p["means"][:, b])  # the donor stays put
        for i in (d, b):  # both halves shrink by exactly 1.6
            np.testing.assert_allclose(np.exp(P["log_scales"][:, i]) * 1.6, np.exp(p["log_scales"][:, b]),
                                       rtol=1e-14)


def test_zero_offset_makes_the_recycled_slot_the_donor():
    p, m, v = _scene([0.005, 0.95], [-3.0, -1.5], seed=3)
    P, _, _, pairs = oracle.relocate(p, m, v, 2, np.zeros((1, 3)))
    assert pairs == [(0, 1)]
    for g in GROUPS:
        np.testing.assert_array_equal(P[g][..., 0], P[g][..., 1])


def test_recycled_offsets_have_the_donors_covariance():
    from scipy.spatial.transform import Rotation
    p, m, v = _scene([0.005, 0.95], [-3.0, -1.5], seed=4)
    rng = np.random.default_rng(5)
    zs = rng.normal(size=(6000, 3))
    offs = np.array([oracle.relocate(p, m, v, 2, z[None])[0]["means"][:, 0] for z in zs]) - p["means"][:, 1]
    w, x, y, zq = p["quats"][:, 1]
    R = Rotation.from_quat([x, y, zq, w]).as_matrix()  # scipy orders (x, y, z, w)
    S2 = np.diag(np.exp(2 * p["log_scales"][:, 1]))
    cov = R @ S2 @ R.T
    np.testing.assert_allclose(np.cov(offs.T), cov, atol=0.06 * np.abs(cov).max())


def test_counts_and_caps():
    p, m, v = _scene([0.01] * 5 + [0.8] * 3, [-1.0] * 8)
    z = np.zeros((10, 3))
    assert len(oracle.relocate(p, m, v, 8, z)[3]) == 3        # fewer donors than dead
    assert len(oracle.relocate(p, m, v, 8, z, max_pairs=2)[3]) == 2
    assert len(oracle.relocate(p, m, v, 8, z[:1])[3]) == 1     # one draw: one pair
    assert [d for d, _ in oracle.relocate(p, m, v, 8, z)[3]] == [0, 1, 2]  # dead in index order
    # equal sizes: donors in index order
    assert [b for _, b in oracle.relocate(p, m, v, 8, z)[3]] == [5, 6, 7]
    # nothing beyond n is looked at
    assert oracle.relocate(p, m, v, 4, z)[3] == []


@pytest.mark.parametrize("o", [0.02, 0.4])
def test_thresholds_are_strict(o):
    p, m, v = _scene([o, 0.9, 0.01], [-1.0, -1.0, -1.0])
    pairs = oracle.relocate(p, m, v, 3, np.zeros((3, 3)))[3]
    assert pairs == [(2, 1)]
