"""The oracle's camera-pose gradient ("How a computer rebuilds a real place ...
Gaussian Splats", section "Forgiving the camera and the light") against what
fixes it independently of its own code:

* float64 central differences of the rendered loss under the pose update
  R <- exp([w]x) R, t <- t + dt (the whole forward re-run at each moved pose);
* the translation equivalence: moving the camera by dt in its own frame moves
  every Gaussian relative to it exactly as translating the scene by R^T dt
  does (positions, view directions), so dL/dt = R sum_i dL/dp_i with the
  oracle's own mean gradients.
"""
import dataclasses
import math

import numpy as np
import pytest

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes


def _skew(v):
    return np.array([[0.0, -v[2], v[1]], [v[2], 0.0, -v[0]], [-v[1], v[0], 0.0]])


def _rotation(axis, angle):
    """exp(angle [axis]x) by Rodrigues' formula (axis a unit vector)."""
    K = _skew(axis)
    return np.eye(3) + math.sin(angle) * K + (1.0 - math.cos(angle)) * (K @ K)


def _posed(cam, R, t):
    """The camera with pose (R, t) in float64 and its centre -R^T t."""
    R = np.asarray(R, np.float64)
    t = np.asarray(t, np.float64)
    return dataclasses.replace(cam, R=R, t=t, campos=-R.T @ t)


def _scene(seed, n=12, W=40, H=32, sh_degree=3):
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
    # the float32 look-at rotation made orthonormal in float64 (nearest rotation)
    U, _, Vt = np.linalg.svd(np.asarray(cam.R, np.float64))
    R = U @ Vt
    cam = _posed(cam, R, -R @ np.array([0.3, -0.2, -0.5]))
    return scenes.make_scene("cam", means, ls, q, logits, sh_degree, sh, [cam], dtype=np.float64)


def _loss_and_structure(scene, cam, target):
    o = oracle.Oracle(scene, cam, camera_f64=True)
    r = o.render()
    L = oracle.loss(r["image"], target, 0.2, with_grad=False)[0]
    return L, (r["n_contrib"].tobytes(), int(r["stats"][1]), int(r["ambiguous"].sum()))


def _pose_gradient(scene, cam, target):
    o = oracle.Oracle(scene, cam, camera_f64=True)
    _, _, _, dimg = oracle.loss(o.render()["image"], target, 0.2)
    g = o.backward(dimg)
    return o.camera_backward(g["screen"]), g


def test_pose_gradient_matches_central_differences():
    h = 1e-6
    checked = skipped = 0
    for seed in (0, 1):
        s = _scene(seed)
        cam = s.cameras[0]
        target = np.random.default_rng(20 + seed).uniform(0, 1, (3, cam.height, cam.width))
        grad, _ = _pose_gradient(s, cam, target)
        assert np.abs(grad).max() > 1e-4
        R0, t0 = np.asarray(cam.R, np.float64), np.asarray(cam.t, np.float64)
        for k in range(6):
            e = np.eye(3)[k % 3]
            if k < 3:
                plus = _posed(cam, _rotation(e, h) @ R0, t0)
                minus = _posed(cam, _rotation(e, -h) @ R0, t0)
            else:
                plus = _posed(cam, R0, t0 + h * e)
                minus = _posed(cam, R0, t0 - h * e)
            Lp, sp = _loss_and_structure(s, plus, target)
            Lm, sm = _loss_and_structure(s, minus, target)
            if sp != sm:  # a threshold decision flipped inside +-h
                skipped += 1
                continue
            num = (Lp - Lm) / (2 * h)
            assert abs(num - grad[k]) <= 1e-6 * abs(num) + 2e-9, (seed, k, num, grad[k])
            checked += 1
    assert checked >= 11 and skipped <= 1


@pytest.mark.parametrize("seed", [2, 3])
def test_translation_gradient_is_the_rotated_sum_of_position_gradients(seed):
    s = _scene(seed)
    cam = s.cameras[0]
    target = np.random.default_rng(30 + seed).uniform(0, 1, (3, cam.height, cam.width))
    grad, g = _pose_gradient(s, cam, target)
    expect = np.asarray(cam.R, np.float64) @ g["means"][:, :s.n].sum(axis=1)
    np.testing.assert_allclose(grad[3:], expect, rtol=1e-9, atol=1e-12)
