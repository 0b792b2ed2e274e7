#!/usr/bin/env python
"""Training-step throughput of the B200 Gaussian-splat rasteriser.

One step = one iteration of the hot path on one camera: preprocess -> tile
sort + forward blend -> L1 + D-SSIM loss -> blend + projection backward ->
Adam on every parameter group, all through the C ABI (include/gs_api.h).

Default workload: the Dense scene (3,000,000 Gaussians from 64 clusters, SH
degree 3, 32 ring cameras at 1920x1080, targets = renders of a perturbed copy
made before timing), cameras drawn from a seeded permutation.

Prints ONE JSON line on rank 0. `--impl reference` times the float64 CPU
oracle on a bounded sample of the same workload instead.
Multi-GPU (torchrun): replicas only - each rank trains its own copy, no
collective on the data path; value = all ranks' iterations / max rank time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "train iters/s (fwd+loss+bwd+Adam), 3M Gaussians @1080p; Mpix/s; % roofline"
UNIT = "iters/s"
PKG_CSRC = os.path.join(ROOT, "gaussian_splatting_differentiable_rasteriser_b200", "csrc")

WORKLOADS = {
    "dense": "dense: 3,000,000 Gaussians (64 clusters, sigma 0.3), SH degree 3, 32 ring cameras "
             "(r = 10) at 1920x1080, f = 1600, targets = renders of a N(0, 0.05^2)-perturbed copy, "
             "seed 0",
    "mid": "mid: 500,000 Gaussians in [-5,5]^3, SH degree 3, 16 ring cameras (r = 15) at 1280x720, "
           "f = 1100, targets = renders of a perturbed copy, seed 0",
    "heavy_tail": "heavy_tail: 6,000,000 Gaussians in 40x10x40, mixture log-scales, SH degree 3, "
                  "32 ring cameras (r = 35) at 1920x1080, targets = renders of a perturbed copy, seed 0",
    "small": "small: 10,000 Gaussians on a unit shell, SH degree 3, one 256x256 camera, "
             "target = renders of a perturbed copy, seed 0",
}

# ncu DRAM traffic (read + write bytes) of kernels per unit of their work, with the
# sha256 (first 12 hex digits) of the source file each figure was taken from. A
# figure whose source has changed since is reported as null. Each was captured with
# ncu on one launch of a smaller case of the same shape and is scaled to a launch
# of the benchmarked workload by the units it processes: the Gaussians (n_pad) for
# the per-Gaussian pass, the (Gaussian, tile) entries for the blend, in which
# traffic grows in proportion.
NCU_TRAFFIC = {
    # Dense-shaped scene of 1.5M Gaussians (3,185,918 entries), one launch of each
    "backward_adam": ((1288.303360e6 + 999.343872e6) / 1_500_000, "gaussians", "9d3c5f2752f4"),
    "blend_backward": ((349.820160e6 + 69.461760e6) / 3_185_918, "entries", "910f1addacf9"),
}


def sha12(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:12]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("sm_max_mhz", 1965.0)), "measured"
    except Exception:
        return 6650.0, 1965.0, "fallback"


class ClockSampler:
    """SM clock and throttle reasons sampled on the host while the GPU works: a
    thread polls NVML (the source nvidia-smi reads) every `period` seconds, from
    start() to stop(). Read-only queries; nothing is set. Falls back to
    `nvidia-smi -lms 50` when the NVML binding is missing."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index, period=0.005):
        self.cuda_index = cuda_index
        self.period = period
        self.rows = []  # (sm MHz, max sm MHz, reason bits)
        self.thread = None
        self.proc = None
        self.path = None
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid if not uuid.startswith("GPU-") else uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        import threading
        try:
            import pynvml
            h = self._nvml_handle()
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._start_smi()
            return
        self.source = "nvml"
        self.stop_flag = threading.Event()

        def poll():
            while not self.stop_flag.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.rows.append((float(sm), float(mx), int(bits)))
                except Exception:
                    pass
                self.stop_flag.wait(self.period)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def _start_smi(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.source = "nvidia-smi"
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        bits = sum(b for (name, b), v in zip(self.REASONS, parts[5:9]) if v.lower() == "active")
                        mx = float(parts[2]) if parts[2].replace(".", "").isdigit() else 0.0
                        self.rows.append((float(parts[1]), mx, bits))
            os.unlink(self.path)
        if not self.rows:
            return out
        out.update(sm_mhz=statistics.median(r[0] for r in self.rows),
                   sm_max_mhz=max(r[1] for r in self.rows),
                   reasons=sorted({name for r in self.rows for name, b in self.REASONS if r[2] & b}),
                   samples=len(self.rows))
        return out


def dist_setup(group_always=False):
    """Rank, world size and device from the launcher's environment; a process group
    when there is more than one rank (or always, for the data-parallel step, whose
    collectives then run on one rank too)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world == 1 and group_always:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(free_port()))
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    if world > 1 or group_always:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def dist_on():
    import torch.distributed as dist
    return dist.is_available() and dist.is_initialized()


def replica_throughput(world, steps, seconds_max):
    """Whole-job iterations per second of `world` replicas that each ran `steps`
    iterations, the slowest taking `seconds_max`."""
    return world * steps / seconds_max


def barrier(world):
    if dist_on():
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ workload
def make_scene(config, gaussians=None):
    """The workload's scene; `gaussians` draws a smaller (or larger) scene of the
    same shape (Dense and Heavy-tail only), for captures that must stay small."""
    from gaussian_splatting_differentiable_rasteriser_b200 import scenes
    if gaussians is None:
        return scenes.CONFIGS[config]()
    if config not in ("dense", "heavy_tail"):
        raise SystemExit("--gaussians applies to the dense and heavy_tail workloads")
    return scenes.CONFIGS[config](n=int(gaussians))


def build_workload(config, device, opacity_rect=False, deterministic=False, loss="l1_dssim",
                   data_parallel=False, exchange="p2p", camera_grad=False, mip_comp=False,
                   gaussians=None, capacity=None):
    import numpy as np
    import torch

    from gaussian_splatting_differentiable_rasteriser_b200 import model, native, scenes

    scene = make_scene(config, gaussians)
    pert = scenes.perturbed(scene, 0.05, seed=1)
    cams = scene.cameras
    W = max(c.width for c in cams)
    H = max(c.height for c in cams)
    m = model.GaussianModel(pert, device=device)
    cap = capacity or max(1 << 20, 8 * scene.n)
    if data_parallel:
        from gaussian_splatting_differentiable_rasteriser_b200.data_parallel import DataParallelTrainStep
        step = DataParallelTrainStep(m, cap, W, H, device=device, opacity_rect=opacity_rect,
                                     deterministic=deterministic, loss=loss, exchange=exchange,
                                     mip_comp=mip_comp)
    else:
        step = model.TrainStep(m, cap, W, H, device=device, opacity_rect=opacity_rect,
                               deterministic=deterministic, loss=loss, mip_comp=mip_comp)
    if camera_grad:
        # every backward also writes the view's pose gradient (6 float64)
        step.camera_grad = torch.zeros(6, dtype=torch.float64, device=device)
        step.ctx.set_camera_grad(step.camera_grad)
    # targets: renders of the perturbed copy (forward only, before any timing)
    targets = torch.empty((len(cams), 3, H, W), dtype=torch.float32, device=device)
    kmax = 0
    for i, cam in enumerate(cams):
        img, _, _ = step.forward(native.camera_struct(cam), cam.height, cam.width)
        targets[i].copy_(img)
        kmax = max(kmax, step.last_entries)
    torch.cuda.synchronize()
    m.load(scene)
    return scene, m, step, targets, kmax


def run_steps(step, cams, targets, sched, start, count):
    for i in range(start, start + count):
        c = int(sched[i % len(sched)])
        step(cams[c], targets[c])


def time_device(step, cams, targets, sched, start, count, world):
    import torch
    barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    run_steps(step, cams, targets, sched, start, count)
    ev1.record()
    torch.cuda.synchronize()
    barrier(world)
    return ev0.elapsed_time(ev1)


BLEND_STAGES = ("blend_forward", "blend_backward")


def profile_stages(step, cams, targets, sched, start, count):
    """Per-stage kernel times (library events) plus Adam (torch events: the
    Adam launches are the only work between them on the current stream). For the
    data-parallel step that stage is "exchange_adam": reduce-scatter, Adam on the
    shard, all-gather.

    The stages are read back after every group of (up to) 5 steps and each
    stage's time is the median over the groups: a stage's events also span any
    time the device waits for the host inside it, and a rare host delay (the
    process descheduled in the middle of a call) would otherwise inflate the
    mean of one stage. Reading back synchronises, so groups keep that to one
    step in five."""
    import torch

    from gaussian_splatting_differentiable_rasteriser_b200 import native

    ctx = step.ctx
    ctx.profile_enable(True)
    ctx.profile_read()
    m = step.model
    ks = []
    group = max(1, min(5, count // 5))
    groups = []
    adam = []
    # one untimed profiled step first, so that no stage's events span a first
    # launch (which can include the loading of the kernel's code)
    for i in range(start - 1, start + count):
        timed = i >= start
        c = int(sched[i % len(sched)])
        cam = cams[c]
        cs = native.camera_struct(cam)
        img, T, nc = step.forward(cs, cam.height, cam.width)
        if timed:
            ks.append(step.last_entries)
        step.compute_loss(img, targets[c], step.dimage)
        if step.fused_adam or getattr(step, "exchange", None) == "views":
            step.backward_and_update(cs, T, nc, step.dimage)
        else:
            m.step_count += 1
            ctx.render_backward(m.params_struct(), cs, T, nc, step.dimage, m.grads_struct())
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            step.update_from_grads()
            e1.record()
            if timed:
                adam.append((e0, e1))
        j = i - start + 1  # timed steps so far
        if not timed or j % group == 0 or j == count:
            torch.cuda.synchronize()
            stages = ctx.profile_read()
            if timed:
                groups.append((stages, j - sum(n for _, n in groups)))
    # The (pixel, Gaussian) pairs of the two blends, for their instruction
    # model, from a second pass over the same cameras with the counting variants
    # of the blend kernels (whose times are not used: the pass above timed the
    # kernels a training run launches).
    ctx.profile_enable(True, count_pairs=True)
    for i in range(start, start + count):
        c = int(sched[i % len(sched)])
        cam = cams[c]
        cs = native.camera_struct(cam)
        img, T, nc = step.forward(cs, cam.height, cam.width)
        step.compute_loss(img, targets[c], step.dimage)
        if step.fused_adam or getattr(step, "exchange", None) == "views":
            step.backward_and_update(cs, T, nc, step.dimage)
        else:
            m.step_count += 1
            ctx.render_backward(m.params_struct(), cs, T, nc, step.dimage, m.grads_struct())
            step.update_from_grads()
    torch.cuda.synchronize()
    counted = ctx.profile_read()
    ctx.profile_enable(False)
    prof = {}
    for name in groups[0][0] if groups else ():
        d = {k: sum(g[name][k] for g, _ in groups) for k in ("launches", "work", "blended")}
        if name in BLEND_STAGES:
            d["work"], d["blended"] = counted[name]["work"], counted[name]["blended"]
        # median over the groups of the stage's time per step, times the steps
        d["ms"] = statistics.median(g[name]["ms"] / n for g, n in groups) * count
        prof[name] = d
    name = "exchange_adam" if hasattr(step, "param_pad") else "adam"
    adam_ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in adam) * len(adam) if adam else 0.0
    adam_launches = len(adam) * step.adam_launches
    prof[name] = {"ms": adam_ms, "launches": adam_launches, "work": adam_launches and count * m.flat.numel()}
    return prof, ks


# FP32 instructions per pixel of the L1 + D-SSIM loss and its gradient in the
# method's separable form, per channel: 3 products (x^2, y^2, xy); 5 moments
# filtered by 11 taps horizontally and vertically (110 FMA); the SSIM map from
# the moments (17) and its three partial derivatives (15); those 3 partials
# filtered back by 11 taps in both directions (66 FMA); dL/dx from them with
# the L1 term and the two loss sums (9): 220 per channel, 660 per pixel.
LOSS_FP32_PER_PIXEL = 3 * (3 + 110 + 17 + 15 + 66 + 9)


def stage_models(scene, sh_k, loss="l1_dssim"):
    """Algorithmic bytes (HBM stages) or FP32-pipe instructions (blend stages and
    the L1 + D-SSIM loss) per unit of work."""
    n_par = 11 + 3 * sh_k
    return {
        # params in (all groups) + 48 B screen + depth + rect + touched + clamp out, per Gaussian
        "preprocess": ("hbm", 4 * n_par + 48 + 4 + 8 + 4 + 1),
        # per item and pass: 32-bit key + 32-bit value read and written (the depth sort's
        # items are the visible Gaussians, the tile sort's the entries)
        "depth_sort": ("hbm", 16),
        "sort": ("hbm", 16),
        # tile key + index written per entry (the 16 B read per visible Gaussian - order,
        # touched, rect - are not counted)
        "duplicate": ("hbm", 8),
        # tile key read (and its neighbour, from cache), per entry
        "ranges": ("hbm", 4),
        # L1 + D-SSIM: FP32 instructions per pixel (issue-bound: its 36 B per pixel of
        # image, target and gradient take a few percent of its time at the HBM peak);
        # Charbonnier: image and target read, gradient written, per pixel (3 channels)
        "loss": ("alu", (LOSS_FP32_PER_PIXEL, 0)) if loss == "l1_dssim" else ("hbm", 36),
        # params + grads read, grads written, raw sums + screen record read, per Gaussian
        "preprocess_backward": ("hbm", 4 * n_par * 3 + 48 + 48 + 5),
        # p, g, m, v read; p, m, v, g = 0 written, per scalar
        "adam": ("hbm", 32),
        # the data-parallel exchange + Adam on one rank (gs_adam_step_reduce with one
        # source, zeroing it): the same 32 B per scalar; with several ranks the stage
        # also holds the two barriers and the NVLink transfers
        "exchange_adam": ("hbm", 32),
        # the views update on one rank, per Gaussian of its range: p, m, v read and
        # written (24 B per scalar), the view's screen record, raw sums and flags
        "views_adam": ("hbm", 24 * n_par + 48 + 48 + 5),
        # fused projection backward + Adam with no accumulated gradient (one view per
        # step): p, m, v read and written, 24 B per scalar of every group, plus the raw
        # screen-gradient sums, the screen record and two flags, per Gaussian
        "backward_adam": ("hbm", 24 * n_par + 48 + 48 + 5),
        # camera-pose gradient, per Gaussian as a visible one reads it: 40 B of
        # geometry parameters, the 48 B screen record, the 48 B raw sums, touched and
        # clamp flags (5 B) and the 192 B of SH coefficients of three coloured channels
        "camera_backward": ("hbm", 40 + 48 + 48 + 5 + 4 * 3 * sh_k),
        # FP32 instructions: 7 per pair the method's walk visits (2 subtractions + 5 for the
        # exponent's quadratic form), plus per blended pair 6 in the forward (weight, 3
        # colour FMAs, transmittance update) and 19 in the backward (T recovery 2,
        # colour dot 3, dL/dalpha 2, weight 1, tail update 1, 3 colour grads, 7 for the
        # six raw sums)
        "blend_forward": ("alu", (7, 6)),
        "blend_backward": ("alu", (7, 19)),
    }


def roofline(prof, scene, hbm_gbs, sm_mhz, loss="l1_dssim"):
    models = stage_models(scene, scene.sh_k, loss)
    per = {}
    for name, d in prof.items():
        if d["launches"] == 0 or name not in models:
            continue
        kind, per_unit = models[name]
        t = d["ms"] / d["launches"] * 1e-3
        units = d["work"] / d["launches"]
        if kind == "hbm":
            achieved = units * per_unit / t / 1e9
            per[name] = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "ms_per_launch": t * 1e3}
        else:
            # FP32 lanes: 148 SMs x 128 lanes x clock (one instruction per lane per cycle)
            peak = 148 * 128 * sm_mhz * 1e6 / 1e12
            per_visit, per_blend = per_unit
            blended = d.get("blended", 0) / d["launches"]
            achieved = (units * per_visit + blended * per_blend) / t / 1e12
            per[name] = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tinst/s",
                         "frac": achieved / peak, "ms_per_launch": t * 1e3}
    return per


# ------------------------------------------------------------- oracle (CPU)
def subset_scene(scene, stride, offset=0):
    """Every stride-th Gaussian of the scene from `offset` (input preparation for a
    bounded sample)."""
    from gaussian_splatting_differentiable_rasteriser_b200 import scenes
    sl = slice(offset, scene.n, stride)
    return scenes.make_scene(scene.name + f"/{stride}+{offset}", scene.means[:, sl], scene.log_scales[:, sl],
                             scene.quats[:, sl], scene.opacity_logits[sl], scene.sh_degree,
                             scene.sh[:, :, sl], scene.cameras)


def host_threads(scene):
    """Threads for the oracle: every CPU this process may run on, capped so that the
    per-thread screen-gradient buffers (n x 9 float64 each) take at most half of
    the free host memory."""
    cpus = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    try:
        import psutil
        free = psutil.virtual_memory().available
    except Exception:
        free = 16 << 30
    per_thread = scene.n * 9 * 8 + (64 << 20)
    return max(1, min(cpus, int(0.5 * free // per_thread)))


class OracleSampler:
    """Estimates the host time of one full training step of the float64 oracle
    from a bounded sample, run on `threads` host threads at once (the oracle's C
    calls release the GIL and only read the shared scene state), part by part,
    each part's wall time scaled by the share of the step it covers:
      preprocess + tile sort of `threads` disjoint subsets, each every
        `stride`-th Gaussian                                    x stride / threads
      render + loss + blend backward of `threads` disjoint bands
        of `rows` pixel rows                                    x height / (threads rows)
      projection backward of `threads` disjoint slices, each
        1/stride of the Gaussians                               x stride / threads
      Adam over `threads` slices of the parameters, each a
        fraction `adam_frac`                                    x 1 / (threads adam_frac)
    The bands and the projection slices use the full scene seen by one camera,
    prepared once outside the timed parts (its preprocess is the one timed on the
    subsets); every output buffer is allocated once. Each thread adds its bands'
    blend backward into a screen-gradient buffer of its own; rows and Gaussians
    written by different threads are disjoint."""

    def __init__(self, scene, cam, target, rows, stride, adam_frac, threads=None):
        import concurrent.futures

        import numpy as np

        import oracle

        self.np, self.oracle = np, oracle
        self.threads = threads or host_threads(scene)
        T = self.threads
        self.pool = concurrent.futures.ThreadPoolExecutor(max_workers=T)
        self.scene, self.adam_frac = scene, adam_frac
        self.stride = max(stride, T)
        self.subs = [subset_scene(scene, self.stride, k) for k in range(T)]
        self.full = oracle.Oracle(scene, cam)
        H, W = cam.height, cam.width
        self.H = H
        self.rows = max(1, min(rows, H // T))
        y_lo = (H - T * self.rows) // 2
        self.bands = [(y_lo + k * self.rows, y_lo + (k + 1) * self.rows) for k in range(T)]
        self.target = np.asarray(target, np.float64)
        self.out = self.full.render_rows(0, 0)  # full-size buffers, rows filled by the bands
        self.dimage = np.zeros((3, H, W))
        self.sg = [np.zeros((scene.n, 9)) for _ in range(T)]
        n = scene.n
        self.grads = dict(means=np.zeros((3, scene.n_pad)), log_scales=np.zeros((3, scene.n_pad)),
                          quats=np.zeros((4, scene.n_pad)), opacity_logits=np.zeros(scene.n_pad),
                          sh=np.zeros((3, scene.sh_k, scene.n_pad)))
        # screen gradients for the projection slices: every touched Gaussian gets a
        # non-zero one, as in a full step where every visible Gaussian is reached
        touched = self.full.preprocess()["touched"] > 0
        per = max(1, n // self.stride)
        lo = max(0, n // 2 - T * per // 2)
        self.slices = [(min(n, lo + k * per), min(n, lo + (k + 1) * per)) for k in range(T)]
        self.sg_slice = np.zeros((n, 9))
        for i0, i1 in self.slices:
            self.sg_slice[i0:i1][touched[i0:i1]] = 1e-3
        total = scene.means.size + scene.log_scales.size + scene.quats.size + \
            scene.opacity_logits.size + scene.sh.size
        cnt = max(1, int(total * adam_frac))
        rng = np.random.default_rng(0)
        self.adam_arrays = [(rng.normal(size=cnt), rng.normal(size=cnt) * 1e-3, np.zeros(cnt), np.zeros(cnt))
                            for _ in range(T)]

    def _band(self, k):
        np, oracle = self.np, self.oracle
        y0, y1 = self.bands[k]
        self.full.render_rows(y0, y1, out=self.out)
        _, _, _, d = oracle.loss(self.out["image"][:, y0:y1, :], self.target[:, y0:y1, :], 0.2)
        self.dimage[:, y0:y1, :] = d
        self.sg[k].fill(0.0)
        self.full.blend_backward_rows(y0, y1, self.dimage, self.sg[k])

    def _run(self, fn):
        list(self.pool.map(fn, range(self.threads)))

    def step(self, cam):
        """One sampled step with camera `cam` for the preprocess part; returns
        (estimated seconds of a full step, wall seconds spent)."""
        oracle = self.oracle
        T = self.threads
        t0 = time.perf_counter()
        self._run(lambda k: oracle.Oracle(self.subs[k], cam))  # preprocess + duplicate + sort + ranges
        t1 = time.perf_counter()
        self._run(self._band)
        t2 = time.perf_counter()
        self._run(lambda k: self.full.project_backward(self.sg_slice, *self.slices[k], self.grads))
        t3 = time.perf_counter()
        self._run(lambda k: oracle.adam(*self.adam_arrays[k], 1e-3, 1))
        t4 = time.perf_counter()
        est = ((t1 - t0) * self.stride / T + (t2 - t1) * self.H / (T * self.rows) +
               (t3 - t2) * self.stride / T + (t4 - t3) / (self.adam_frac * T))
        return est, t4 - t0

    def fractions(self):
        """Share of each part of a full step that one sampled step covers."""
        T = self.threads
        return {"preprocess_sort": T / self.stride, "render_loss_blend_backward": T * self.rows / self.H,
                "projection_backward": T / self.stride, "adam": T * self.adam_frac}

    def describe(self):
        T = self.threads
        return (f"float64 oracle on {T} host threads at once: preprocess + tile sort of {T} subsets, each "
                f"every {self.stride}th of {self.scene.n} Gaussians, x {self.stride}/{T}; render + loss + "
                f"blend backward of {T} bands of {self.rows} rows, x height/{T * self.rows}; projection "
                f"backward of {T} slices of 1/{self.stride} of the Gaussians, x {self.stride}/{T}; Adam on "
                f"{T} slices of 1/{round(1 / self.adam_frac)} of the parameters, "
                f"x {round(1 / self.adam_frac)}/{T}; the step time is an estimate from these parts")

    def close(self):
        self.pool.shutdown()


def cpu_baseline(scene, cams, targets_host, sched):
    """One sampled step of the oracle on the host's cores (our arm's reported
    baseline), after one untimed sampled step that warms the threads' memory."""
    c = int(sched[0])
    t0 = time.perf_counter()
    s = OracleSampler(scene, cams[c], targets_host[c], rows=48, stride=8, adam_frac=1 / 64)
    s.step(cams[c])
    prep = time.perf_counter() - t0
    est, spent = s.step(cams[c])
    s.close()
    return {"value": 1.0 / est, "unit": UNIT, "cores": s.threads, "kind": "oracle",
            "sample": "1 step: " + s.describe(), "estimated": True, "sample_fraction": s.fractions(),
            "seconds_spent": spent, "seconds_setup": prep}


# ------------------------------------------------------------------- arms
def main_ours(args):
    import numpy as np
    import torch

    import __graft_entry__

    world, rank, local = dist_setup(group_always=args.parallel == "dp")
    if rank == 0:
        __graft_entry__.build()
    barrier(world)
    from gaussian_splatting_differentiable_rasteriser_b200 import native, scenes

    native.load()
    device = f"cuda:{local}"
    scene, m, step, targets, kmax = build_workload(args.config, device, args.rect == "opacity",
                                                   args.deterministic, args.loss, args.parallel == "dp",
                                                   args.exchange, args.camera_grad, args.mip,
                                                   args.gaussians, args.capacity)
    cams = scene.cameras
    sched = scenes.camera_schedule(len(cams), args.warmup + args.steps, seed=rank)
    # clocks are sampled from the start of the warm-up to the end of the timed region
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    run_steps(step, cams, targets, sched, 0, args.warmup)
    torch.cuda.synchronize()
    ms = time_device(step, cams, targets, sched, args.warmup, args.steps, world)
    clk = clocks.stop()
    clk["window"] = "warm-up and timed steps"
    ms = max_over_ranks(ms, world)
    ms_per_step = ms / args.steps
    value = replica_throughput(world, args.steps, ms / 1e3)
    H, W = cams[0].height, cams[0].width

    # per-stage kernel times for the roofline (separate, profiled pass over the same steps)
    prof, ks = profile_stages(step, cams, targets, sched, args.warmup, args.steps)
    hbm_gbs, sm_max, peak_kind = peaks()
    per = roofline(prof, scene, hbm_gbs, clk["sm_mhz"] or sm_max, args.loss)
    dominant = max((k for k in prof if prof[k]["launches"]), key=lambda k: prof[k]["ms"])
    rf = dict(per.get(dominant, {}))
    rf.pop("ms_per_launch", None)
    rf["kernel"] = dominant
    rf["peak_source"] = peak_kind
    src = {"blend_forward": "blend.cu", "blend_backward": "blend.cu", "adam": "adam.cu",
           "preprocess": "preprocess.cu", "sort": "sort.cu", "depth_sort": "sort.cu", "loss": "loss.cu",
           "preprocess_backward": "preprocess_backward.cu",
           "backward_adam": "preprocess_backward.cu", "exchange_adam": "adam_reduce.cu",
           "views_adam": "views_adam.cu",
           "camera_backward": "camera_backward.cu"}.get(dominant)
    tr = NCU_TRAFFIC.get(dominant)
    rf["traffic"] = None
    if tr and src and sha12(os.path.join(PKG_CSRC, src)) == tr[2]:
        units = scene.n_pad if tr[1] == "gaussians" else (statistics.mean(ks) if ks else 0)
        rf["traffic"] = tr[0] * units

    # launches of our kernels in the timed region: the profiler counts every kernel a
    # context launches (over the same steps), plus gs_adam_step per group when the
    # separate path is used
    steps_p = max(1, args.steps)
    per_step = (sum(prof[k]["launches"] for k in prof if k not in ("adam", "exchange_adam")) / steps_p +
                (0 if step.fused_adam else step.adam_launches))
    gpu_launches = int(round(per_step * args.steps))

    # end to end: target streamed from pinned host memory each step, loss read back
    e2e = None
    if not args.no_e2e:
        e2e = e2e_run(step, cams, targets, sched, args, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(scene, cams, targets.cpu().numpy(), sched)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.config] + (f"; {scene.n} Gaussians drawn instead"
                                                             if args.gaussians else ""),
                       "gaussians": scene.n,
                       "width": W, "height": H, "cameras": len(cams),
                       "parallelism": (("data-parallel: one camera per rank; each rank's screen-space view "
                                        "read by the owner of each Gaussian, projection backward and Adam "
                                        "fused (gs_adam_step_views)" if args.exchange == "views" else
                                        "data-parallel: one camera per rank; gradient exchange fused with "
                                        "the sharded Adam over peer memory (gs_adam_step_reduce)"
                                        if args.exchange == "p2p" else
                                        "data-parallel: one camera per rank; NCCL reduce-scatter, "
                                        "sharded Adam, NCCL all-gather") if args.parallel == "dp"
                                       else "replicas" if world > 1 else "single-gpu"),
                       "tile_rect": "3 sigma" if args.rect == "3sigma" else "opacity-aware",
                       "gradient_sums": "fixed-point (deterministic)" if args.deterministic else "float32 atomics",
                       "loss": "L1 + D-SSIM (lambda 0.2)" if args.loss == "l1_dssim" else "Charbonnier + exposure",
                       "camera_grad": bool(args.camera_grad),
                       "mip_compensation": bool(args.mip),
                       "l2": "inputs larger than L2: 2.1 GB of parameter and moment state (p, m, v) "
                             "streamed every step" if args.config == "dense" else "see workload",
                       "entries_per_step": int(statistics.mean(ks)) if ks else None},
            "mpix_per_s": value * W * H / 1e6,
            "roofline": rf,
            "stages": {k: {"ms_per_step": prof[k]["ms"] / steps_p,
                           "share": prof[k]["ms"] / max(1e-9, sum(v["ms"] for v in prof.values())),
                           **({"frac": per[k]["frac"], "bound": per[k]["bound"],
                               "achieved": per[k]["achieved"], "unit": per[k]["unit"]}
                              if k in per else {})}
                       for k in prof if prof[k]["launches"]},
            "e2e": e2e, "gpu_launches": gpu_launches, "clocks": clk, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if hasattr(step, "close"):
        step.close()
    if dist_on():
        import torch.distributed as dist
        dist.destroy_process_group()


def e2e_run(step, cams, targets, sched, args, world):
    """Same steps through the public API with the target of every step copied
    from pinned host memory (double-buffered on a copy stream, overlapped with the
    previous step's work) and each step's loss read back to the host (on the copy
    stream, as soon as the loss kernel has run)."""
    import torch

    from gaussian_splatting_differentiable_rasteriser_b200 import native

    host_t = targets.cpu().pin_memory()
    dev_t = [torch.empty_like(targets[0]) for _ in range(2)]
    copy_stream = torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    loss_ready = [torch.cuda.Event() for _ in range(2)]
    loss_read = [torch.cuda.Event() for _ in range(2)]
    loss_host = torch.empty((2, 3), dtype=torch.float64).pin_memory()
    m = step.model
    n = args.steps
    start = args.warmup
    losses = []
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    c0 = int(sched[start % len(sched)])
    with torch.cuda.stream(copy_stream):
        dev_t[0].copy_(host_t[c0], non_blocking=True)
        copied[0].record(copy_stream)
    compute = torch.cuda.current_stream()
    for j in range(n):
        i = start + j
        c = int(sched[i % len(sched)])
        cam = cams[c]
        cs = native.camera_struct(cam)
        # Cross-stream waits sit at the step boundary, where the step's chain
        # of kernels starts anyway: this step's target has landed (it was copied
        # during the previous step), and the previous loss has been read out of
        # the loss buffer before this step's loss kernel rewrites it.
        compute.wait_event(copied[j % 2])
        if j > 0:
            compute.wait_event(loss_read[(j - 1) % 2])
        img, T, nc = step.forward(cs, cam.height, cam.width)  # waits for all earlier work
        if j > 0:
            loss_read[(j - 1) % 2].synchronize()
            losses.append(float(loss_host[(j - 1) % 2, 0]))
        if j + 1 < n:
            cn = int(sched[(i + 1) % len(sched)])
            with torch.cuda.stream(copy_stream):
                dev_t[(j + 1) % 2].copy_(host_t[cn], non_blocking=True)
                copied[(j + 1) % 2].record(copy_stream)
        step.compute_loss(img, dev_t[j % 2], step.dimage)
        # the loss goes to the host on the copy stream, off the compute stream
        loss_ready[j % 2].record(compute)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(loss_ready[j % 2])
            loss_host[j % 2].copy_(step.loss[:3], non_blocking=True)
            loss_read[j % 2].record(copy_stream)
        step.backward_and_update(cs, T, nc, step.dimage)
    torch.cuda.synchronize()
    losses.append(float(loss_host[(n - 1) % 2, 0]))
    dt = time.perf_counter() - t0
    dt = max_over_ranks(dt, world)
    barrier(world)
    assert len(losses) == n
    H, W = cams[0].height, cams[0].width
    return {"value": replica_throughput(world, n, dt), "unit": UNIT, "h2d_bytes_per_step": 3 * H * W * 4,
            "d2h_bytes_per_step": 3 * 8 + 24, "last_loss": losses[-1]}


def main_reference(args):
    """The float64 CPU oracle on the same workload, on every host core, each step a
    bounded sample (OracleSampler: one 2-row band and one 1/256 subset per thread)
    so that the whole run stays within minutes. The value is an estimate of the
    full step from the sampled parts ("estimated": true). Rank 0 alone runs; other
    ranks exit without work."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from gaussian_splatting_differentiable_rasteriser_b200 import scenes

    oracle.lib()
    scene = scenes.CONFIGS[args.config]()
    pert = scenes.perturbed(scene, 0.05, seed=1)
    cams = scene.cameras
    sched = scenes.camera_schedule(len(cams), args.warmup + args.steps, seed=0)
    H, W = cams[0].height, cams[0].width
    c0 = int(sched[0])
    threads = host_threads(scene)
    rows = max(1, min(2, H // threads))
    # the target of the sampled bands: the perturbed copy's render of those rows,
    # on the same threads
    import concurrent.futures

    import numpy as np
    ref = oracle.Oracle(pert, cams[c0])
    target = ref.render_rows(0, 0)
    y_lo = (H - threads * rows) // 2
    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda k: ref.render_rows(y_lo + k * rows, y_lo + (k + 1) * rows, out=target),
                    range(threads)))
    target = np.array(target["image"])
    del ref
    sampler = OracleSampler(scene, cams[c0], target, rows=rows, stride=256, adam_frac=1 / 4096,
                            threads=threads)
    est, spent = [], 0.0
    for i in range(args.warmup + args.steps):
        e, s = sampler.step(cams[int(sched[i])])
        if i >= args.warmup:
            est.append(e)
            spent += s
    sampler.close()
    value = len(est) / sum(est)
    cpu = {"value": value, "unit": UNIT, "cores": sampler.threads, "kind": "oracle",
           "sample": "per step: " + sampler.describe(), "estimated": True,
           "sample_fraction": sampler.fractions(), "seconds_spent": spent}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOADS[args.config] + (f"; {scene.n} Gaussians drawn instead"
                                                             if args.gaussians else ""),
                       "gaussians": scene.n, "width": W,
                       "height": H, "cameras": len(cams), "parallelism": "cpu"},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def densify_inputs(scene, seed=0):
    """Seeded synthetic density-control inputs for a scene: view counts 0..4,
    accumulated gradient norms (exponential per view), N(0,1) split draws, and
    thresholds placing about 10% of the Gaussians above the gradient cut and
    half of those above the scale cut; opacity prune at 0.005."""
    import numpy as np
    rng = np.random.default_rng(seed)
    n_pad = scene.n_pad
    count = rng.integers(0, 5, n_pad).astype(np.int32)
    accum = (rng.exponential(1.0, n_pad) * count).astype(np.float32)
    normals = rng.normal(size=(n_pad, 2, 3)).astype(np.float32)
    avg = np.where(count > 0, accum / np.maximum(count, 1), 0.0)[: scene.n]
    grad_thr = float(np.quantile(avg[count[: scene.n] > 0], 0.9))
    scale_thr = float(np.exp(np.median(scene.log_scales[:, : scene.n].max(axis=0))))
    return accum, count, normals, grad_thr, scale_thr, 0.005


def main_densify(args):
    """Throughput of one densification pass (gs_densify) on the workload's
    Gaussians with synthetic statistics, against the HBM roofline (parameters
    and moments read, statistics read, new set written); the oracle timed on a
    1/200 sample of the Gaussians beside it."""
    import numpy as np
    import torch

    import __graft_entry__

    world, rank, local = dist_setup()
    if rank == 0:
        __graft_entry__.build()
    barrier(world)
    from gaussian_splatting_differentiable_rasteriser_b200 import model, native, scenes
    from gaussian_splatting_differentiable_rasteriser_b200.scenes import GROUP_NAMES

    native.load()
    device = f"cuda:{local}"
    scene = scenes.CONFIGS[args.config]()
    accum, count, normals, gthr, sthr, mop = densify_inputs(scene)
    m = model.GaussianModel(scene, device=device)
    m.m_flat.normal_(0, 1e-3)
    m.v_flat.uniform_(0, 1e-6)
    out = model.GaussianModel(scene, device=device)  # output storage, re-strided below
    cap = (2 * scene.n + 3) // 4 * 4
    out._alloc(cap)
    ctx = native.Context(scene.n_pad, 16, 16, 16)
    d_acc = torch.from_numpy(accum).to(device)
    d_cnt = torch.from_numpy(count).to(device)
    d_nrm = torch.from_numpy(normals).to(device)
    p_in, (m_in, v_in) = m.params_struct(), m.moments_structs()
    p_out, (m_out, v_out) = out._struct(out.params), out.moments_structs()

    def one():
        return ctx.densify(p_in, m_in, v_in, d_acc, d_cnt, d_nrm, gthr, sthr, mop, p_out, m_out, v_out, cap)

    for _ in range(args.warmup):
        n_out = one()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        n_out = one()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    value = replica_throughput(world, args.steps, ms / 1e3)
    n = scene.n
    planes = 11 + 3 * scene.sh_k
    splits = n_out - n  # each split adds one net Gaussian, each clone one, each prune removes one
    algo_bytes = n * (planes * 12 + 8) + n_out * planes * 12
    hbm_gbs, _, peak_kind = peaks()
    achieved = algo_bytes * value / world / 1e9
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        sl = slice(0, n, 200)
        sub = {k: getattr(scene, k)[..., sl].astype(np.float64) for k in GROUP_NAMES}
        zeros = {k: np.zeros_like(x) for k, x in sub.items()}
        k_n = sub["opacity_logits"].shape[-1]
        t0 = time.perf_counter()
        oracle.densify(sub, zeros, zeros, k_n, accum[sl][:k_n], count[sl][:k_n], normals[sl][:k_n], gthr, sthr,
                       mop)
        est = (time.perf_counter() - t0) * n / k_n
        cpu = {"value": 1.0 / est, "unit": "passes/s", "cores": 1, "kind": "oracle",
               "sample": f"float64 oracle densify of every 200th of {n} Gaussians, scaled by 200; single-threaded"}
    if rank == 0:
        line = {"metric": "densify passes/s (prune/clone/split with compaction)", "value": value,
                "unit": "passes/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOADS[args.config] + "; synthetic densification statistics",
                           "gaussians_in": n, "gaussians_out": int(n_out), "net_added": int(splits),
                           "grad_threshold": gthr, "scale_threshold": sthr, "min_opacity": mop},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                             "frac": achieved / hbm_gbs, "traffic": None, "peak_source": peak_kind,
                             "bytes_per_pass": algo_bytes},
                "e2e": None, "gpu_launches": 3 * args.steps, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main_relocate(args):
    """Time of one recycling pass (gs_relocate) on the workload's Gaussians with
    their own opacities (dead < 0.02, donors > 0.4), one normal draw per dead
    Gaussian; the parameters are restored between passes, outside the timed
    region. Roofline: HBM bytes of the classification, the donors' 4-pass sort and
    the pair writes; the oracle timed on a 1/200 sample beside it."""
    import numpy as np
    import torch

    import __graft_entry__

    world, rank, local = dist_setup()
    if rank == 0:
        __graft_entry__.build()
    barrier(world)
    from gaussian_splatting_differentiable_rasteriser_b200 import model, native, scenes
    from gaussian_splatting_differentiable_rasteriser_b200.scenes import GROUP_NAMES

    native.load()
    device = f"cuda:{local}"
    scene = scenes.CONFIGS[args.config]()
    m = model.GaussianModel(scene, device=device)
    m.m_flat.normal_(0, 1e-3)
    m.v_flat.uniform_(0, 1e-6)
    backup = [t.clone() for t in (m.flat, m.m_flat, m.v_flat)]
    logits = scene.opacity_logits[:scene.n].astype(np.float64)
    dead = int((logits < math.log(0.02 / 0.98)).sum())
    donors = int((logits > math.log(0.4 / 0.6)).sum())
    normals = torch.from_numpy(np.random.default_rng(7).normal(size=(max(dead, 1), 3)).astype(np.float32)).to(device)
    ctx = native.Context(scene.n_pad, 16, 16, 16)
    total_ms, pairs = 0.0, 0
    for it in range(args.warmup + args.steps):
        for t, b in zip((m.flat, m.m_flat, m.v_flat), backup):
            t.copy_(b)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pairs = m.relocate(ctx, normals)
        e1.record()
        torch.cuda.synchronize()
        if it >= args.warmup:
            total_ms += e0.elapsed_time(e1)
    ms = max_over_ranks(total_ms, world)
    value = replica_throughput(world, args.steps, ms / 1e3)
    n = scene.n
    planes = 11 + 3 * scene.sh_k
    algo_bytes = n * 16 + donors * (8 + 4 * 16) + dead * 4 + pairs * planes * 4 * 6
    hbm_gbs, _, peak_kind = peaks()
    achieved = algo_bytes * value / world / 1e9
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        sl = slice(0, n, 200)
        sub = {k: getattr(scene, k)[..., sl].astype(np.float64) for k in GROUP_NAMES}
        zeros = {k: np.zeros_like(x) for k, x in sub.items()}
        k_n = sub["opacity_logits"].shape[-1]
        t0 = time.perf_counter()
        oracle.relocate(sub, zeros, zeros, k_n, normals.cpu().numpy())
        est = (time.perf_counter() - t0) * n / k_n
        cpu = {"value": 1.0 / est, "unit": "passes/s", "cores": 1, "kind": "oracle",
               "sample": f"float64 oracle relocate of every 200th of {n} Gaussians, scaled by 200; single-threaded"}
    if rank == 0:
        line = {"metric": "relocate passes/s (dead Gaussians recycled onto the largest donors)", "value": value,
                "unit": "passes/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": WORKLOADS[args.config], "gaussians": n, "dead": dead, "donors": donors,
                           "pairs": int(pairs), "dead_opacity": 0.02, "donor_opacity": 0.4},
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                             "frac": achieved / hbm_gbs, "traffic": None, "peak_source": peak_kind,
                             "bytes_per_pass": algo_bytes},
                "e2e": None, "gpu_launches": 10 * args.steps, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", choices=tuple(WORKLOADS), default="dense")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rect", choices=("3sigma", "opacity"), default="3sigma",
                    help="tile rect: the 3-sigma radius, or the opacity-aware one (same image, fewer entries)")
    ap.add_argument("--deterministic", action="store_true",
                    help="fixed-point gradient atomics (bitwise-reproducible backward)")
    ap.add_argument("--loss", choices=("l1_dssim", "charbonnier"), default="l1_dssim",
                    help="photometric loss of the step")
    ap.add_argument("--parallel", choices=("replicas", "dp"), default="replicas",
                    help="N>1: independent replicas (default), or data-parallel training over cameras "
                         "(one camera per rank per iteration; value counts camera-iterations)")
    ap.add_argument("--exchange", choices=("views", "p2p", "nccl"), default="views",
                    help="--parallel dp: each rank's screen-space view read by the owner of each Gaussian "
                         "(projection backward + Adam fused), the gradient exchange fused with Adam over peer "
                         "memory, or NCCL collectives")
    ap.add_argument("--gaussians", type=int, default=None,
                    help="draw this many Gaussians instead (dense, heavy_tail): a same-shaped smaller case")
    ap.add_argument("--capacity", type=int, default=None,
                    help="(Gaussian, tile) entry capacity of the context (default 8 per Gaussian)")
    ap.add_argument("--mip", action="store_true",
                    help="opacities times the Mip-Splatting compensation factor")
    ap.add_argument("--camera-grad", action="store_true",
                    help="each backward also computes the view's camera-pose gradient")
    ap.add_argument("--op", choices=("step", "densify", "relocate"), default="step",
                    help="the training step (default), one densification pass or one recycling pass")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        main_reference(args)
    elif args.op == "densify":
        main_densify(args)
    elif args.op == "relocate":
        main_relocate(args)
    else:
        main_ours(args)


if __name__ == "__main__":
    main()
