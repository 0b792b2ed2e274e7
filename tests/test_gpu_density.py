"""Adaptive density control on the GPU against the float64 oracle: the
screen-gradient statistics the backward accumulates, one densification pass
(prune / clone / split, stream-compacted) and the opacity reset."""
import numpy as np
import pytest

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gs():
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import model, native
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    native.load()
    return native, model


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    return t.detach().cpu().numpy()


def rel_l2(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


@pytest.mark.parametrize("fused", [False, True])
def test_backward_accumulates_densify_statistics(gs, fused):
    native, model = gs
    s = scenes.small()
    cam = s.cameras[0]
    m = model.GaussianModel(s)
    st = model.TrainStep(m, 200_000, cam.width, cam.height, fused_adam=fused)
    accum = torch.zeros(s.n_pad, device="cuda")
    count = torch.zeros(s.n_pad, dtype=torch.int32, device="cuda")
    st.ctx.set_densify_stats(accum, count)
    target = scenes.uniform_image(cam.height, cam.width, seed=3)
    for _ in range(2):  # two views of the same camera: the statistics double
        m.load(s)
        st(cam, dev(target))
    torch.cuda.synchronize()
    st.ctx.set_densify_stats(None, None)
    o = oracle.Oracle(s, cam)
    r = o.render()
    _, _, _, dimg = oracle.loss(r["image"].astype(np.float32), target, 0.2)
    ref = o.backward(dimg)
    norm, cnt = oracle.densify_stats(ref["screen"], o.preprocess()["touched"])
    np.testing.assert_array_equal(host(count)[: s.n], 2 * cnt)
    assert rel_l2(host(accum)[: s.n], 2 * norm) < 1e-3


def _inputs(n=3000, seed=0):
    rng = np.random.default_rng(seed)
    s = scenes.small(seed=5)
    n_pad = s.n_pad
    p = {k: getattr(s, k).astype(np.float32) for k in scenes.GROUP_NAMES}
    p["opacity_logits"] = rng.normal(0, 3, n_pad).astype(np.float32)
    p["log_scales"] = np.log(rng.uniform(0.005, 0.2, (3, n_pad))).astype(np.float32)
    m = {k: rng.normal(0, 1e-3, v.shape).astype(np.float32) for k, v in p.items()}
    v = {k: rng.uniform(0, 1e-6, val.shape).astype(np.float32) for k, val in p.items()}
    count = rng.integers(0, 5, n_pad).astype(np.uint32)
    accum = (rng.exponential(1.0, n_pad) * count).astype(np.float32)
    normals = rng.normal(size=(n_pad, 2, 3)).astype(np.float32)
    return s, p, m, v, accum, count, normals


def test_densify_matches_oracle(gs):
    native, model = gs
    s, p, m, v, accum, count, normals = _inputs()
    n = s.n
    gt, st_, mo = np.float32(1.5), np.float32(0.05), np.float32(0.02)
    ref_p, ref_m, ref_v, ref_n = oracle.densify(
        {k: x.astype(np.float64) for k, x in p.items()}, {k: x.astype(np.float64) for k, x in m.items()},
        {k: x.astype(np.float64) for k, x in v.items()}, n, accum, count, normals,
        float(gt), float(st_), float(mo))
    assert 0 < ref_n != n
    gm = model.GaussianModel(s)
    for k in scenes.GROUP_NAMES:
        gm.params[k].copy_(dev(p[k]))
        gm.m[k].copy_(dev(m[k]))
        gm.v[k].copy_(dev(v[k]))
    ctx = native.Context(s.n_pad, 16, 16, 16)
    n_out = gm.densify(ctx, dev(accum), dev(count.astype(np.int32), torch.int32), dev(normals), gt, st_, mo)
    torch.cuda.synchronize()
    assert n_out == ref_n
    for k in scenes.GROUP_NAMES:
        got_p = host(gm.params[k])[..., :n_out].astype(np.float64)
        got_m = host(gm.m[k])[..., :n_out].astype(np.float64)
        got_v = host(gm.v[k])[..., :n_out].astype(np.float64)
        if k in ("means", "log_scales"):
            np.testing.assert_allclose(got_p, ref_p[k], rtol=1e-6, atol=1e-6, err_msg=k)
        else:
            np.testing.assert_array_equal(got_p, ref_p[k], err_msg=k)
        np.testing.assert_array_equal(got_m, ref_m[k], err_msg=k)
        np.testing.assert_array_equal(got_v, ref_v[k], err_msg=k)
    # copied columns (kept Gaussians and clones) are exact in every group: the
    # columns whose log-scales match the oracle's exactly are the copies, and
    # their means match exactly too
    ls_got = host(gm.params["log_scales"])[:, :n_out].astype(np.float64)
    copies = np.all(ls_got == ref_p["log_scales"], axis=0)
    assert copies.sum() >= n_out // 2
    np.testing.assert_array_equal(host(gm.params["means"])[:, :n_out][:, copies].astype(np.float64),
                                  ref_p["means"][:, copies])


def test_densify_capacity_and_arguments(gs):
    native, model = gs
    s, p, m, v, accum, count, normals = _inputs()
    gm = model.GaussianModel(s)
    ctx = native.Context(s.n_pad, 16, 16, 16)
    with pytest.raises(native.GsError) as e:
        gm.densify(ctx, dev(accum), dev(count.astype(np.int32), torch.int32), dev(normals), 1.5, 0.05,
                   0.02, capacity=4)
    assert e.value.status == native.GS_ERR_CAPACITY
    gm = model.GaussianModel(s)
    with pytest.raises(native.GsError):
        gm.densify(ctx, dev(accum), dev(count.astype(np.int32), torch.int32), dev(normals), 1.5, 0.05, 1.5)


def test_opacity_reset_matches_oracle(gs):
    native, _ = gs
    rng = np.random.default_rng(2)
    logits = rng.normal(0, 4, 1001).astype(np.float32)
    m = rng.normal(size=1001).astype(np.float32)
    v = rng.uniform(size=1001).astype(np.float32)
    tl, tm, tv = dev(logits), dev(m), dev(v)
    native.opacity_reset(tl, tm, tv, 0.01)
    torch.cuda.synchronize()
    ref, rm, rv = oracle.opacity_reset(logits.astype(np.float64), m, v, 0.01)
    np.testing.assert_allclose(host(tl), ref, rtol=0, atol=1e-6)
    below = logits.astype(np.float64) <= ref
    np.testing.assert_array_equal(host(tl)[below], logits[below])
    assert not host(tm).any() and not host(tv).any()


@pytest.mark.parametrize("rows", [40, 400])
def test_relocation_matches_oracle(gs, rows):
    """gs_relocate in place against the oracle's recycling: the same pairs (the
    first `rows` pairs, or every dead Gaussian when there are fewer), the
    recycled and shrunk Gaussians within float32 rounding, every other slot
    bit for bit as before, and the reshaped Gaussians' moments at zero."""
    native, model = gs
    s = scenes.small()
    m = model.GaussianModel(s)
    ctx = native.Context(s.n_pad, 1 << 16, 64, 64)
    gen = torch.Generator(device="cuda").manual_seed(1)
    m.m_flat.normal_(0.0, 1e-3, generator=gen)
    m.v_flat.uniform_(0.0, 1e-6, generator=gen)
    groups = scenes.GROUP_NAMES
    p0 = {k: host(m.params[k]).copy() for k in groups}
    m0 = {k: host(m.m[k]).copy() for k in groups}
    v0 = {k: host(m.v[k]).copy() for k in groups}
    normals = np.random.default_rng(3).normal(size=(rows, 3)).astype(np.float32)
    pairs = m.relocate(ctx, torch.from_numpy(normals).cuda())
    torch.cuda.synchronize()
    rp, rm, rv, ref_pairs = oracle.relocate(p0, m0, v0, s.n, normals)
    assert pairs == len(ref_pairs) > 0
    if rows == 40:
        assert pairs == 40
    touched = sorted({i for pr in ref_pairs for i in pr})
    other = np.setdiff1d(np.arange(s.n_pad), touched)
    for k in groups:
        gp, gm, gv = host(m.params[k]), host(m.m[k]), host(m.v[k])
        np.testing.assert_array_equal(gp[..., other], p0[k][..., other])
        np.testing.assert_array_equal(gm[..., other], m0[k][..., other])
        np.testing.assert_array_equal(gv[..., other], v0[k][..., other])
        np.testing.assert_allclose(gp[..., touched], rp[k][..., touched], rtol=1e-6, atol=1e-6)
        assert not gm[..., touched].any() and not gv[..., touched].any()
