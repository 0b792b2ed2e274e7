"""The data-parallel step on the GPU.

* gs_adam_step_reduce with every rank's buffers on this one GPU (one launch per
  rank's shard, as each rank would issue it; the launches wait on nothing, so
  this is the multi-rank data path run in order): every rank's parameters end
  identical, equal bit for bit to Adam on the float32 rank-ordered mean
  gradient, and within float32 rounding of the float64 oracle's Adam.
* One source with zeroing is gs_adam_step, bit for bit.
* The whole DataParallelTrainStep with a one-rank NCCL group, for the three
  exchanges, and with two processes on one GPU over gloo (the exchange reading
  and writing the other process's memory through CUDA IPC): with the
  fixed-point (order-independent) gradient sums the parameters are those of a
  single-GPU step on the mean gradient of the ranks' cameras - bitwise for the
  gradient exchanges, to float32 rounding for the views exchange (whose
  replicas are bitwise equal among themselves).
* The views exchange with 1-3 emulated ranks on one GPU.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

import oracle
from gaussian_splatting_differentiable_rasteriser_b200 import scenes

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def native():
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import native as nat
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    nat.load()
    return nat


def assert_close_params(a, b, frac=0.999):
    """Two parameter (or moment) buffers from the same operations in different
    kernels: nearly every scalar within float32 rounding; none off by more than
    the size of a few Adam steps (an Adam step normalises the gradient, so a
    gradient within rounding of zero may step either way)."""
    a = a.detach().cpu().numpy().astype(np.float64)
    b = b.detach().cpu().numpy().astype(np.float64)
    close = np.abs(a - b) <= 1e-6 + 1e-6 * np.abs(b)
    assert close.mean() >= frac, close.mean()
    assert np.abs(a - b).max() <= 1e-2 + 1e-5 * np.abs(b).max()


def test_one_source_with_zeroing_is_adam_step(native):
    g = torch.Generator().manual_seed(0)
    for count, off in ((4096, 0), (1003, 0), (1000, 1)):
        p, gr, m, v = (torch.randn(count + 8, generator=g).cuda() for _ in range(4))
        v.abs_()
        ref = [t.clone() for t in (p, gr, m, v)]
        sl = slice(off, off + count)
        native.adam_step(ref[0][sl], ref[1][sl], ref[2][sl], ref[3][sl], 1e-3, 3)
        native.adam_step_reduce(p[sl], m[sl], v[sl], [gr[sl].data_ptr()], [], 1e-3, 3, zero_grads=True)
        torch.cuda.synchronize()
        for a, b in zip((p, gr, m, v), ref):
            assert torch.equal(a, b)


@pytest.mark.parametrize("world,count,aligned", [(2, 8192, True), (3, 3001, False), (4, 10_000, False),
                                                 (8, 4 * 1237, True)])
def test_emulated_ranks_reduce_adam_allgather(native, world, count, aligned):
    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    from gaussian_splatting_differentiable_rasteriser_b200.scenes import GROUP_NAMES
    rng = np.random.default_rng(world)
    # five groups summing to count: ragged sizes (the scalar kernel), or multiples of
    # 4 floats (16-byte-aligned pieces: the float4 kernel)
    if aligned:
        cuts = 4 * np.sort(rng.choice(np.arange(1, count // 4), 4, replace=False))
    else:
        cuts = np.sort(rng.choice(np.arange(1, count), 4, replace=False))
    sizes = np.diff(np.concatenate([[0], cuts, [count]]))
    slices, off = {}, 0
    for k, n in zip(GROUP_NAMES, sizes):
        slices[k] = slice(off, off + int(n))
        off += int(n)
    lrs = dict(zip(GROUP_NAMES, (1.6e-4, 5e-3, 1e-3, 5e-2, 2.5e-3)))
    pad = dp.padded_size(count, world)
    p0 = rng.normal(size=count).astype(np.float32)
    m0 = rng.normal(0, 1e-2, count).astype(np.float32)
    v0 = rng.uniform(0, 1e-4, count).astype(np.float32)
    grads = [rng.normal(0, 1e-2, count).astype(np.float32) for _ in range(world)]
    step = 4
    params, gbufs, ms, vs = [], [], [], []
    for r in range(world):
        t = torch.zeros(pad, device="cuda")
        t[:count] = torch.from_numpy(p0)
        params.append(t)
        t = torch.zeros(pad, device="cuda")
        t[:count] = torch.from_numpy(grads[r])
        gbufs.append(t)
        ms.append(torch.zeros(pad, device="cuda"))
        vs.append(torch.zeros(pad, device="cuda"))
        ms[r][:count] = torch.from_numpy(m0)
        vs[r][:count] = torch.from_numpy(v0)
    pp = [t.data_ptr() for t in params]
    gp = [t.data_ptr() for t in gbufs]
    for r in range(world):
        for k, a, b, gsrc, copies in dp.p2p_pieces(slices, count, world, r, pp, gp):
            native.adam_step_reduce(params[r][a:b], ms[r][a:b], vs[r][a:b], gsrc, copies, lrs[k], step)
    torch.cuda.synchronize()
    out = [t[:count].cpu().numpy() for t in params]
    for r in range(1, world):
        np.testing.assert_array_equal(out[r], out[0])
    for t in params:
        assert not t[count:].any()
    for r in range(world):  # sources are read, not zeroed
        np.testing.assert_array_equal(gbufs[r][:count].cpu().numpy(), grads[r])
    # bitwise: the float32 rank-ordered sum times 1/world, then gs_adam_step
    gsum = torch.from_numpy(grads[0]).cuda()
    for r in range(1, world):
        gsum = gsum + torch.from_numpy(grads[r]).cuda()
    gsum = gsum * np.float32(1.0 / world)
    rp, rm, rv = (torch.from_numpy(x).cuda() for x in (p0, m0, v0))
    for k in GROUP_NAMES:
        s = slices[k]
        native.adam_step(rp[s], gsum[s], rm[s], rv[s], lrs[k], step)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out[0], rp.cpu().numpy())
    m_all = np.zeros(count, np.float32)
    for r in range(world):
        lo, hi = dp.shard_bounds(count, world, r)
        m_all[lo:min(hi, count)] = ms[r][lo:min(hi, count)].cpu().numpy()
    np.testing.assert_array_equal(m_all, rm.cpu().numpy())
    # the float64 oracle's Adam on the exact mean gradient
    gmean = np.mean(np.stack(grads).astype(np.float64), axis=0)
    for k in GROUP_NAMES:
        s = slices[k]
        op, _, om, ov = oracle.adam(p0[s], gmean[s], m0[s], v0[s], lrs[k], step)
        np.testing.assert_allclose(out[0][s], op, rtol=0, atol=2e-6 + 1e-6 * lrs[k] / 1e-3)
        np.testing.assert_allclose(m_all[s], om, rtol=1e-5, atol=1e-9)


@pytest.mark.parametrize("exchange", ["views", "p2p", "nccl"])
def test_one_rank_nccl_step_equals_the_single_gpu_step(native, exchange):
    import torch.distributed as dist

    from gaussian_splatting_differentiable_rasteriser_b200 import model
    from gaussian_splatting_differentiable_rasteriser_b200.data_parallel import DataParallelTrainStep
    scene = scenes.small()
    cam = scene.cameras[0]
    target = torch.from_numpy(scenes.uniform_image(cam.height, cam.width, seed=3)).cuda()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        ma, mb = model.GaussianModel(scene), model.GaussianModel(scene)
        cap = 1 << 20
        a = DataParallelTrainStep(ma, cap, cam.width, cam.height, deterministic=True, exchange=exchange)
        b = model.TrainStep(mb, cap, cam.width, cam.height, fused_adam=False, deterministic=True)
        assert a.world == 1 and a.adam_launches == (1 if exchange == "views" else len(scenes.GROUP_NAMES))
        for _ in range(3):
            la, lb = a(cam, target), b(cam, target)
        torch.cuda.synchronize()
        if exchange == "views":
            # the same operations in another kernel: the parameters agree up to
            # float32 rounding after each step, so the losses of the later steps
            # agree to about that relative precision
            np.testing.assert_allclose(la.cpu().numpy(), lb.cpu().numpy(), rtol=1e-7, atol=1e-12)
            assert_close_params(ma.flat, mb.flat)
            assert_close_params(ma.m_flat, mb.m_flat)
        else:
            np.testing.assert_array_equal(la.cpu().numpy(), lb.cpu().numpy())
            assert torch.equal(ma.flat, mb.flat) and torch.equal(ma.m_flat, mb.m_flat)
            assert torch.equal(ma.v_flat, mb.v_flat)
        if exchange != "views":
            assert not a.grad_pad.any() and not a.param_pad[ma.flat.numel():].any()
        assert not torch.equal(ma.flat, model.GaussianModel(scene).flat)  # the step moved them
        a.close()
    finally:
        dist.destroy_process_group()


def _rank(rank, world, port, out_dir, steps, exchange="p2p"):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from gaussian_splatting_differentiable_rasteriser_b200 import model
    from gaussian_splatting_differentiable_rasteriser_b200 import native as nat
    from gaussian_splatting_differentiable_rasteriser_b200.data_parallel import DataParallelTrainStep
    torch.cuda.set_device(0)
    nat.load()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    scene = scenes.small()
    cams = [scenes.look_at((3.0 * np.sin(a), 0.3, -3.0 * np.cos(a)), (0.0, 0.0, 0.0), 256, 256, 256.0)
            for a in (0.0, 0.4)]
    targets = [torch.from_numpy(scenes.uniform_image(256, 256, seed=10 + r)).cuda() for r in range(world)]
    m = model.GaussianModel(scene)
    s = DataParallelTrainStep(m, 1 << 20, 256, 256, deterministic=True, exchange=exchange)
    assert len(s._peer_maps) == (2 if exchange == "p2p" else 6) * (world - 1)
    for _ in range(steps):
        s(cams[rank], targets[rank])
    torch.cuda.synchronize()
    np.save(os.path.join(out_dir, f"p{rank}.npy"), m.flat.cpu().numpy())
    np.save(os.path.join(out_dir, f"m{rank}.npy"), m.m_flat.cpu().numpy())
    if rank == 0:
        # the same iterations on one process: each camera's gradient on its own (from a
        # zero buffer, as on its rank), summed in rank order, halved (exact), then Adam
        # per group
        r = model.GaussianModel(scene)
        t = model.TrainStep(r, 1 << 20, 256, 256, fused_adam=False, deterministic=True)
        for _ in range(steps):
            r.step_count += 1
            gsum = None
            for c in range(world):
                cs = nat.camera_struct(cams[c])
                img, T, nc = t.forward(cs, 256, 256)
                t.compute_loss(img, targets[c], t.dimage)
                r.grad_flat.zero_()
                t.ctx.render_backward(r.params_struct(), cs, T, nc, t.dimage, r.grads_struct())
                gsum = r.grad_flat.clone() if gsum is None else gsum + r.grad_flat
            r.grad_flat.copy_(gsum * 0.5)
            t.update_from_grads()
        torch.cuda.synchronize()
        np.save(os.path.join(out_dir, "ref_p.npy"), r.flat.cpu().numpy())
        np.save(os.path.join(out_dir, "ref_m.npy"), r.m_flat.cpu().numpy())
    s.close()
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("exchange", ["p2p", "views"])
def test_two_processes_on_one_gpu_exchange(native, tmp_path, exchange):
    """Two processes on one GPU over gloo, each mapping the other's buffers through
    CUDA IPC: p2p reads the other's gradient and writes its parameters; views reads
    the other's screen sums, flags and camera and writes its parameters."""
    import torch.multiprocessing as mp

    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    world, steps = 2, 2
    mp.start_processes(_rank, args=(world, free_port(), str(tmp_path), steps, exchange), nprocs=world, join=True,
                       start_method="spawn")
    p0, p1, ref = (np.load(tmp_path / f) for f in ("p0.npy", "p1.npy", "ref_p.npy"))
    np.testing.assert_array_equal(p0, p1)  # the replicas are the same bits
    ref_m = np.load(tmp_path / "ref_m.npy")
    total = ref_m.size
    if exchange == "p2p":
        np.testing.assert_array_equal(p0, ref)
    else:
        assert_close_params(torch.from_numpy(p0), torch.from_numpy(ref))
    for r in range(world):
        if exchange == "p2p":
            lo, hi = dp.shard_bounds(total, world, r)
            np.testing.assert_array_equal(np.load(tmp_path / f"m{r}.npy")[lo:hi], ref_m[lo:hi])
        else:  # each rank holds the moments of its own Gaussians in every plane
            n_pad = scenes.small().n_pad
            lo, hi = dp.gaussian_bounds(n_pad, world, r)
            col = np.arange(total) % n_pad
            own = (col >= lo) & (col < hi)
            assert_close_params(torch.from_numpy(np.load(tmp_path / f"m{r}.npy")[own]), torch.from_numpy(ref_m[own]))


@pytest.mark.parametrize("world", [1, 2, 3])
def test_views_exchange_emulated_ranks_equal_the_gradient_exchange(native, world):
    """Each emulated rank (a context and a parameter replica on this GPU) renders its
    own camera and runs only the blend backward; then every rank's
    gs_adam_step_views updates its Gaussians from all the views and writes them
    into every replica (the launches wait on nothing, so this is the multi-rank
    data path run in order). With fixed-point (order-independent) screen sums the
    replicas end with the same bits, equal up to float32 rounding to the gradient
    exchange (each view's full gradient, summed in rank order, times 1 / ranks,
    then Adam) and within float32 rounding of the float64 oracle's Adam on the
    mean gradient."""
    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    from gaussian_splatting_differentiable_rasteriser_b200 import model
    scene = scenes.small()
    cams = [scenes.look_at((3.0 * np.sin(a), 0.3 * a, -3.0 * np.cos(a)), (0.0, 0.0, 0.0), 256, 256, 256.0)
            for a in (0.0, 0.5, -0.7)][:world]
    targets = [scenes.uniform_image(256, 256, seed=30 + r) for r in range(world)]
    lrs = [1.6e-4, 5e-3, 1e-3, 5e-2, 2.5e-3]
    step = 3
    g = torch.Generator().manual_seed(7)
    reps, ctxs, dimgs = [], [], []
    for r in range(world):
        m = model.GaussianModel(scene)
        if r == 0:
            m0 = (torch.randn(m.m_flat.numel(), generator=g) * 1e-3).cuda()
            v0 = (torch.rand(m.v_flat.numel(), generator=g) * 1e-6).cuda()
        m.m_flat.copy_(m0)
        m.v_flat.copy_(v0)
        t = model.TrainStep(m, 1 << 20, 256, 256, fused_adam=False, deterministic=True)
        cs = native.camera_struct(cams[r])
        img, T, nc = t.forward(cs, 256, 256)
        t.compute_loss(img, torch.from_numpy(targets[r]).cuda(), t.dimage)
        reps.append((m, t, cs, T, nc))
        dimgs.append(t.dimage.clone())
    # the gradient exchange's result, on a separate replica
    ref = model.GaussianModel(scene)
    ref.m_flat.copy_(m0)
    ref.v_flat.copy_(v0)
    gsum = None
    for r, (m, t, cs, T, nc) in enumerate(reps):
        m.grad_flat.zero_()
        t.ctx.render_backward(m.params_struct(), cs, T, nc, dimgs[r], m.grads_struct())
        gsum = m.grad_flat.clone() if gsum is None else gsum + m.grad_flat
        m.grad_flat.zero_()
    ref.grad_flat.copy_(gsum * np.float32(1.0 / world))
    for k, lr in zip(scenes.GROUP_NAMES, lrs):
        native.adam_step(ref.params[k], ref.grads[k], ref.m[k], ref.v[k], lr, step)
    # the views exchange
    for r, (m, t, cs, T, nc) in enumerate(reps):
        t.ctx.render_backward_screen(m.params_struct(), cs, T, nc, dimgs[r])
    views = [t.ctx.view() for (_, t, _, _, _) in reps]
    for r, (m, t, cs, T, nc) in enumerate(reps):
        lo, hi = dp.gaussian_bounds(m.n_pad, world, r)
        copies = [o[0]._struct(o[0].params) for q, o in enumerate(reps) if q != r]
        em, ev = m.moments_structs()
        t.ctx.adam_step_views(m.params_struct(), views, lo, hi, copies, em, ev, lrs, step)
    torch.cuda.synchronize()
    for m, *_ in reps:
        assert torch.equal(m.flat, reps[0][0].flat)
    assert_close_params(reps[0][0].flat, ref.flat)
    n_pad = ref.n_pad
    col = torch.arange(ref.m_flat.numel(), device="cuda") % n_pad
    for r, (m, *_) in enumerate(reps):
        lo, hi = dp.gaussian_bounds(n_pad, world, r)
        own = (col >= lo) & (col < hi)
        assert_close_params(m.m_flat[own], ref.m_flat[own])
        assert_close_params(m.v_flat[own], ref.v_flat[own])
    assert not torch.equal(ref.flat, model.GaussianModel(scene).flat)
    # against the float64 oracle: Adam on the mean of the views' gradients
    gm = {k: np.zeros(ref.params[k].shape) for k in scenes.GROUP_NAMES}
    for r in range(world):
        o = oracle.Oracle(scene, cams[r])
        gr = o.backward(dimgs[r].cpu().numpy().astype(np.float64))
        for k in scenes.GROUP_NAMES:
            gm[k] += gr[k] / world
    p0 = model.GaussianModel(scene)
    for k, lr in zip(scenes.GROUP_NAMES, lrs):
        sl = ref.slices[k]
        want = oracle.adam(p0.params[k].cpu().numpy(), gm[k], m0[sl].cpu().numpy(), v0[sl].cpu().numpy(), lr,
                           step)[0].reshape(ref.params[k].shape)
        got = ref.params[k].cpu().numpy().astype(np.float64)
        real = (np.arange(got.size) % n_pad < scene.n).reshape(got.shape)
        assert np.mean(np.abs(got - want)[real] <= 2e-6 + 1e-3 * lr) > 0.999, k

