"""The benchmark's multi-rank host logic on CPU with the gloo backend, world
size 2: process-group set-up from the launcher's environment, the barrier,
the max-over-ranks timing and the whole-job aggregate of independent replicas,
and the reference arm under the launcher (rank 0 prints the one line, the
other rank exits without work); plus the roofline arithmetic, the scaling
of the ncu traffic figures, and the profiled pass taking its stage times from
the production kernels and the blends' pair counts from a separate counting
pass (a fake context, no GPU)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    bench.barrier(w)
    # each replica's own device time; the job is as slow as its slowest rank
    local_ms = 100.0 + 50.0 * rank
    ms = bench.max_over_ranks(local_ms, w)
    value = bench.replica_throughput(w, 10, ms / 1e3)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"ms": ms, "value": value}, f)
    bench.barrier(w)
    dist.destroy_process_group()


def test_replicas_take_the_slowest_rank(tmp_path):
    import torch.multiprocessing as mp
    port = free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    outs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for o in outs:
        assert o["ms"] == 150.0
        assert o["value"] == pytest.approx(2 * 10 / 0.150)


def test_reference_arm_under_the_launcher_prints_once():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--config", "small", "--gpus", "2", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_roofline_arithmetic():
    """achieved = algorithmic bytes (or FP32 instructions) per launch / launch time;
    frac = achieved / peak; the fused pass moves 59 x 24 + 101 B per Gaussian."""
    sys.path.insert(0, ROOT)
    import types

    import bench
    scene = types.SimpleNamespace(sh_k=16, n=3_000_000, n_pad=3_000_000)
    prof = {"backward_adam": {"ms": 2.0, "launches": 2, "work": 6_000_000, "blended": 0},
            "blend_forward": {"ms": 1.0, "launches": 2, "work": 4_000_000, "blended": 1_000_000},
            "scan": {"ms": 0.1, "launches": 1, "work": 0, "blended": 0}}
    per = bench.roofline(prof, scene, 6555.2, 1965.0)
    assert "scan" not in per  # no model, no roofline entry
    ba = per["backward_adam"]
    assert ba["bound"] == "hbm" and ba["unit"] == "GB/s"
    assert ba["achieved"] == pytest.approx(3_000_000 * (59 * 24 + 101) / 1e-3 / 1e9)
    assert ba["frac"] == pytest.approx(ba["achieved"] / 6555.2)
    bf = per["blend_forward"]
    peak = 148 * 128 * 1965.0e6 / 1e12
    assert bf["bound"] == "alu" and bf["peak"] == pytest.approx(peak)
    assert bf["achieved"] == pytest.approx((2_000_000 * 7 + 500_000 * 6) / 0.5e-3 / 1e12)


def test_traffic_figures_scale_per_unit_of_work():
    sys.path.insert(0, ROOT)
    import bench
    per_g, unit, _ = bench.NCU_TRAFFIC["backward_adam"]
    assert unit == "gaussians"
    # on the captured case (a Dense-shaped scene of 1.5M Gaussians, 3,185,918 entries)
    # each figure gives back the launch's read + write bytes
    assert per_g * 1_500_000 == pytest.approx(1288.303360e6 + 999.343872e6)
    # and it is close to the fused pass's algorithmic bytes per Gaussian (24 B per scalar + 101 B)
    assert per_g == pytest.approx(24 * 59 + 101, rel=0.01)
    per_e, unit, _ = bench.NCU_TRAFFIC["blend_backward"]
    assert unit == "entries" and per_e * 3_185_918 == pytest.approx(349.820160e6 + 69.461760e6)


class _FakeCtx:
    """Stands in for a library context: times (fixed per-stage figures) when
    profiling is on, counts the blends' pairs only when asked to."""

    def __init__(self):
        self.modes = []
        self.steps = 0

    def profile_enable(self, on=True, count_pairs=False):
        self.modes.append((on, count_pairs))
        self.steps = 0

    def profile_read(self):
        on, count = self.modes[-1] if self.modes else (False, False)
        n, self.steps = self.steps, 0
        out = {}
        for name, ms in (("blend_forward", 0.5), ("blend_backward", 0.7), ("backward_adam", 0.9)):
            blend = name.startswith("blend")
            # the counting variants are slower: their times must not be used
            t = ms * (3.0 if count and blend else 1.0)
            out[name] = {"ms": t * n, "launches": n, "work": (1000 * n if count and blend else 7 * n),
                         "blended": (200 * n if count and blend else 0)}
        return out


class _FakeStep:
    fused_adam = True
    adam_launches = 0

    def __init__(self):
        self.ctx = _FakeCtx()
        self.model = type("M", (), {"step_count": 0})()
        self.dimage = None
        self.last_entries = 123

    def forward(self, cs, h, w):
        self.ctx.steps += 1
        return None, None, None

    def compute_loss(self, img, target, dimage):
        pass

    def backward_and_update(self, cs, T, nc, dimage):
        pass


def test_profiled_stage_times_come_from_the_timing_pass_and_pair_counts_from_the_counting_pass(monkeypatch):
    sys.path.insert(0, ROOT)
    import torch

    import bench
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(native, "camera_struct", lambda cam: cam)
    step = _FakeStep()
    cam = type("C", (), {"height": 4, "width": 4})()
    prof, ks = bench.profile_stages(step, [cam], [None], [0], start=1, count=10)
    # timing pass first (production kernels), then the counting pass, then off
    assert step.ctx.modes == [(True, False), (True, True), (False, False)]
    assert prof["blend_forward"]["ms"] == pytest.approx(0.5 * 10)
    assert prof["blend_backward"]["ms"] == pytest.approx(0.7 * 10)
    assert prof["blend_backward"]["work"] == 1000 * 10 and prof["blend_backward"]["blended"] == 200 * 10
    # stages without a counting variant keep the timing pass's work units
    assert prof["backward_adam"]["work"] == 7 * 10 and prof["backward_adam"]["ms"] == pytest.approx(9.0)
    assert ks == [123] * 10
    assert prof["adam"]["launches"] == 0  # the fused pass: no separate Adam launches
