"""The data-parallel exchange step on the host with the gloo backend, world
size 2: the reduce-scatter / sharded Adam / all-gather leaves both ranks with
the parameters of one Adam step on the batch-mean gradient, as the float64
oracle computes it on the whole buffer; the sharding arithmetic and the peer
addresses of the fused exchange; and a rank that fails before the exchange
makes its peer's collective fail instead of hang."""
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shards_cover_the_buffer_once_and_stay_aligned():
    sys.path.insert(0, ROOT)
    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    for total in (1, 7, 4096, 10_003):
        for world in (1, 2, 3, 8):
            b = [dp.shard_bounds(total, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == dp.padded_size(total, world) >= total
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            assert all(lo % dp.ALIGN == 0 and (hi - lo) == b[0][1] - b[0][0] for lo, hi in b)


def _slices(sizes):
    out, off = {}, 0
    for k, n in sizes.items():
        out[k] = slice(off, off + n)
        off += n
    return out, off


def _rank(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    from gaussian_splatting_differentiable_rasteriser_b200.scenes import GROUP_NAMES
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    sizes = dict(zip(GROUP_NAMES, (30, 30, 40, 10, 130)))
    slices, total = _slices(sizes)
    lrs = dict(zip(GROUP_NAMES, (1e-3, 2e-3, 5e-4, 1e-2, 1e-3)))
    rng = np.random.default_rng(0)
    p0 = rng.normal(size=total).astype(np.float32)
    grads = [rng.normal(0, 1e-2, total).astype(np.float32) for _ in range(world)]
    pad = dp.padded_size(total, world)
    param_pad = torch.zeros(pad)
    param_pad[:total] = torch.from_numpy(p0)
    grad_pad = torch.zeros(pad)
    grad_pad[:total] = torch.from_numpy(grads[rank])
    m = torch.zeros(total)
    v = torch.zeros(total)

    def adam(p, g, mm, vv, k):  # the float64 oracle as the update, on the host
        rp, _, rm, rv = oracle.adam(p.numpy(), g.numpy(), mm.numpy(), vv.numpy(), lrs[k], 1)
        p.copy_(torch.from_numpy(rp.astype(np.float32)))
        mm.copy_(torch.from_numpy(rm.astype(np.float32)))
        vv.copy_(torch.from_numpy(rv.astype(np.float32)))
        g.zero_()

    dp.exchange_and_update(grad_pad, param_pad, m, v, slices, total, world, rank, adam)
    assert not grad_pad.any()
    np.save(os.path.join(out_dir, f"p{rank}.npy"), param_pad[:total].numpy())
    if rank == 0:
        gmean = (grads[0].astype(np.float64) + grads[1].astype(np.float64)) / 2
        ref = np.empty(total)
        for k in GROUP_NAMES:
            s = slices[k]
            ref[s] = oracle.adam(p0[s], gmean[s].astype(np.float32), np.zeros(sizes[k]), np.zeros(sizes[k]),
                                 lrs[k], 1)[0]
        np.save(os.path.join(out_dir, "ref.npy"), ref)
    dist.barrier()
    dist.destroy_process_group()


def test_exchange_matches_adam_on_the_batch_mean_gradient(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_rank, args=(2, free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    p0, p1, ref = (np.load(tmp_path / f) for f in ("p0.npy", "p1.npy", "ref.npy"))
    np.testing.assert_array_equal(p0, p1)
    # the shard's mean gradient is float32 (g0 + g1) / 2: within a few float32 ulps of lr-sized steps
    np.testing.assert_allclose(p0, ref, rtol=0, atol=1e-6)


def test_p2p_pieces_address_every_rank_at_the_shard():
    sys.path.insert(0, ROOT)
    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    from gaussian_splatting_differentiable_rasteriser_b200.scenes import GROUP_NAMES
    sizes = dict(zip(GROUP_NAMES, (300, 300, 400, 100, 4800)))
    slices, total = _slices(sizes)
    world = 4
    pp = [1 << 40 | r << 32 for r in range(world)]
    gp = [1 << 41 | r << 32 for r in range(world)]
    covered = np.zeros(total, int)
    for rank in range(world):
        lo, hi = dp.shard_bounds(total, world, rank)
        for k, a, b, gsrc, copies in dp.p2p_pieces(slices, total, world, rank, pp, gp):
            assert lo <= a < b <= hi and slices[k].start <= a and b <= slices[k].stop
            assert gsrc == [g + 4 * a for g in gp]
            assert copies == [p + 4 * a for r, p in enumerate(pp) if r != rank]
            covered[a:b] += 1
    assert (covered == 1).all()


def _rank_fails(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    from gaussian_splatting_differentiable_rasteriser_b200.scenes import GROUP_NAMES
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=10))
    slices, total = _slices(dict(zip(GROUP_NAMES, (8, 8, 8, 4, 36))))
    pad = dp.padded_size(total, world)
    status = "ok"
    try:
        if rank == 1:
            raise RuntimeError("this rank's backward failed")  # leaves before the exchange
        dp.exchange_and_update(torch.ones(pad), torch.zeros(pad), torch.zeros(total), torch.zeros(total),
                               slices, total, world, rank, lambda *a: None)
    except Exception as e:  # noqa: BLE001 - the test records what each rank saw
        status = f"error: {type(e).__name__}"
    open(os.path.join(out_dir, f"status{rank}.txt"), "w").write(status)
    if rank == 1:
        os._exit(0)  # leaves without a clean shutdown, as a crashed rank does
    try:
        dist.destroy_process_group()
    except Exception:  # noqa: BLE001
        pass


def test_a_rank_that_fails_before_the_exchange_makes_the_others_fail_not_hang(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_fails, args=(2, free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    assert (tmp_path / "status1.txt").read_text().startswith("error")
    assert (tmp_path / "status0.txt").read_text().startswith("error")


def _rank_state(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    from gaussian_splatting_differentiable_rasteriser_b200 import model, scenes
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    m = model.GaussianModel(scenes.small(), device="cpu")
    total = m.flat.numel()
    g = torch.Generator().manual_seed(3)
    M = torch.randn(total, generator=g)
    V = torch.rand(total, generator=g)
    # after data-parallel steps a rank's moments are right on its own shard only
    lo, hi = dp.shard_bounds(total, world, rank)
    m.m_flat.fill_(100.0 + rank)
    m.v_flat.fill_(-1.0 - rank)
    m.m_flat[lo:min(hi, total)] = M[lo:min(hi, total)]
    m.v_flat[lo:min(hi, total)] = V[lo:min(hi, total)]
    m.attach_storage(m.flat, m.grad_flat, owner=object())
    refused = False
    try:
        m.state_dict()
    except RuntimeError:
        refused = True
    assert refused, "a model whose storage a data-parallel step owns must not save its partial moments"
    mf = dp.gather_shards(m.m_flat, total, world, rank)
    vf = dp.gather_shards(m.v_flat, total, world, rank)
    state = m.state_dict(m_flat=mf, v_flat=vf)
    torch.save(state, os.path.join(out_dir, f"state{rank}.pt"))
    dist.barrier()
    if rank == 0:
        torch.save({"M": M, "V": V}, os.path.join(out_dir, "truth.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_checkpoint_gathers_every_ranks_moments(tmp_path):
    """Each rank updates the Adam moments of its own shard only; the checkpoint of a
    data-parallel model must hold every shard's moments (gathered), on every rank,
    and restore them into a fresh single-GPU model."""
    import torch
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    from gaussian_splatting_differentiable_rasteriser_b200 import model, scenes
    mp.start_processes(_rank_state, args=(2, free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    truth = torch.load(tmp_path / "truth.pt")
    s0, s1 = torch.load(tmp_path / "state0.pt"), torch.load(tmp_path / "state1.pt")
    for s in (s0, s1):
        assert torch.equal(s["m_flat"], truth["M"]) and torch.equal(s["v_flat"], truth["V"])
    fresh = model.GaussianModel(scenes.small(seed=1), device="cpu")
    fresh.load_state_dict(s0)
    assert torch.equal(fresh.m_flat, truth["M"]) and torch.equal(fresh.v_flat, truth["V"])


def test_an_owned_model_refuses_a_size_change_and_bad_states():
    import pytest
    import torch
    sys.path.insert(0, ROOT)
    from gaussian_splatting_differentiable_rasteriser_b200 import model, scenes
    small = model.GaussianModel(scenes.small(), device="cpu")
    sc = scenes.small()
    sl = slice(0, 4096)
    other = model.GaussianModel(scenes.make_scene("small/4096", sc.means[:, sl], sc.log_scales[:, sl],
                                                  sc.quats[:, sl], sc.opacity_logits[sl], sc.sh_degree,
                                                  sc.sh[:, :, sl], sc.cameras), device="cpu")
    owned = model.GaussianModel(scenes.small(), device="cpu")
    owned.attach_storage(owned.flat, owned.grad_flat, owner=object())
    with pytest.raises(RuntimeError):
        owned.load_state_dict(other.state_dict())
    owned.load_state_dict(small.state_dict())  # same size: allowed
    bad = small.state_dict()
    bad["n"] = bad["n_pad"] + 1
    with pytest.raises(ValueError):
        small.load_state_dict(bad)
    bad = small.state_dict()
    bad["m_flat"] = bad["m_flat"][:-4]
    with pytest.raises(ValueError):
        small.load_state_dict(bad)
    assert torch.equal(owned.flat, small.flat)


def _rank_gaussian_gather(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    n_pad, planes = 1004, 7
    truth = torch.randn(planes * n_pad, generator=torch.Generator().manual_seed(5))
    lo, hi = dp.gaussian_bounds(n_pad, world, rank)
    col = torch.arange(truth.numel()) % n_pad
    mine = torch.where((col >= lo) & (col < hi), truth, torch.full_like(truth, 1e9 + rank))
    full = dp.gather_gaussian_shards(mine, n_pad, world, rank)
    torch.save(full, os.path.join(out_dir, f"g{rank}.pt"))
    if rank == 0:
        torch.save(truth, os.path.join(out_dir, "truth.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_gaussian_ranges_cover_every_gaussian_once_and_gather_exactly(tmp_path):
    """The "views" exchange owns whole Gaussians: every rank's range is a multiple of
    4 columns, the ranges tile [0, n_pad) once, and gathering each rank's own
    columns of every plane gives back the full buffer bit for bit (gloo, 2 and 3
    ranks)."""
    import torch
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    from gaussian_splatting_differentiable_rasteriser_b200 import data_parallel as dp
    for n_pad in (4, 1004, 3_000_000):
        for world in (1, 2, 3, 8):
            b = [dp.gaussian_bounds(n_pad, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n_pad
            assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
            assert all(lo % 4 == 0 and hi % 4 == 0 and lo <= hi for lo, hi in b)
    for world in (2, 3):
        mp.start_processes(_rank_gaussian_gather, args=(world, free_port(), str(tmp_path)), nprocs=world,
                           join=True, start_method="spawn")
        truth = torch.load(tmp_path / "truth.pt")
        for r in range(world):
            assert torch.equal(torch.load(tmp_path / f"g{r}.pt"), truth)
