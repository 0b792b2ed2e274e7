"""The oracle's Charbonnier + exposure loss against what the page and the
mathematics fix: zero at a perfect match, the mean-L1 limit as delta -> 0, a
slope bounded by the gain for outliers, and gradients equal to central
differences of the loss itself."""
import numpy as np

import oracle


def _case(seed=0, H=7, W=9):
    rng = np.random.default_rng(seed)
    x = rng.uniform(0, 1, (3, H, W))
    y = np.clip(x + rng.normal(0, 0.2, x.shape), 0, 1)
    return x, y, np.array([1.1, 0.9, 1.05]), np.array([0.02, -0.01, 0.0])


def test_zero_at_a_perfect_match():
    x, _, _, _ = _case()
    loss, d, dg, db = oracle.charbonnier_loss(x, x, [1, 1, 1], [0, 0, 0])
    assert loss == 0.0
    assert not d.any() and not dg.any() and not db.any()


def test_small_delta_limit_is_the_channel_summed_mean_l1():
    x, y, g, b = _case()
    loss, _, _, _ = oracle.charbonnier_loss(x, y, g, b, delta=1e-9)
    err = g.reshape(3, 1, 1) * x + b.reshape(3, 1, 1) - y
    assert abs(loss - np.abs(err).sum(axis=0).mean()) < 1e-8


def test_outlier_slope_is_bounded_by_the_gain():
    x, y, g, b = _case()
    y[0, 0, 0] = 50.0
    _, d, _, _ = oracle.charbonnier_loss(x, y, g, b)
    P = x.shape[1] * x.shape[2]
    assert np.all(np.abs(d) * P <= g.reshape(3, 1, 1) + 1e-12)
    assert abs(d[0, 0, 0] * P + g[0]) < 1e-3  # saturated at -gain


def test_gradients_match_central_differences():
    x, y, g, b = _case(seed=3)
    _, d, dg, db = oracle.charbonnier_loss(x, y, g, b)
    h = 1e-6
    f = lambda xx, gg, bb: oracle.charbonnier_loss(xx, y, gg, bb)[0]
    for idx in [(0, 0, 0), (1, 3, 4), (2, 6, 8)]:
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        assert abs((f(xp, g, b) - f(xm, g, b)) / (2 * h) - d[idx]) < 1e-7
    for c in range(3):
        e = np.zeros(3)
        e[c] = h
        assert abs((f(x, g + e, b) - f(x, g - e, b)) / (2 * h) - dg[c]) < 1e-7
        assert abs((f(x, g, b + e) - f(x, g, b - e)) / (2 * h) - db[c]) < 1e-7
