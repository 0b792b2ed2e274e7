"""Data-parallel training over cameras, one process per GPU.

Each rank holds a replica of the Gaussians and renders its own camera of the
iteration's batch (the training loop of "How a computer rebuilds a real place
... Gaussian Splats", section "Per step", with one photo per rank). The one
exchange step is the gradient: a reduce-scatter leaves each rank the batch-mean
gradient of its contiguous shard of the flat parameter buffer, each rank runs
Adam on its shard only (the shard's moments are the only ones it updates), and
an all-gather gives every rank the updated parameters. The collectives are
torch.distributed's (NCCL over NVLink / NVSwitch on GPUs, gloo on the host for
tests); the rendering, the backward and Adam are the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import native
from .model import TrainStep
from .scenes import GROUP_NAMES

ALIGN = 4  # floats: shard boundaries keep 16-byte alignment


def padded_size(total: int, world: int) -> int:
    """Smallest size >= total that splits into `world` equal shards of a multiple of ALIGN floats."""
    unit = world * ALIGN
    return (total + unit - 1) // unit * unit


def shard_bounds(total: int, world: int, rank: int):
    """[lo, hi) of rank's shard of a flat buffer of `total` floats (padded to equal shards)."""
    per = padded_size(total, world) // world
    return rank * per, (rank + 1) * per


def group_pieces(slices: dict, lo: int, hi: int):
    """The parts of each parameter group (given as flat slices) that fall inside [lo, hi):
    [(group, start, stop)] in flat coordinates."""
    out = []
    for k in GROUP_NAMES:
        s = slices[k]
        a, b = max(s.start, lo), min(s.stop, hi)
        if a < b:
            out.append((k, a, b))
    return out


def exchange_and_update(grad_pad, param_pad, m_flat, v_flat, slices, total, world, rank, adam_fn, group=None):
    """The exchange step of one data-parallel iteration.

    grad_pad / param_pad: flat buffers of padded_size(total, world) floats
    holding this rank's gradient and the (identical) parameters. After the call
    every rank holds the parameters updated by Adam with the batch-mean
    gradient; grad_pad is zeroed. adam_fn(param, grad, m, v, group_name) updates
    one contiguous piece in place (and zeroes its gradient)."""
    lo, hi = shard_bounds(total, world, rank)
    shard = torch.empty(hi - lo, dtype=grad_pad.dtype, device=grad_pad.device)
    collective = dist.is_available() and dist.is_initialized()
    if collective:
        dist.reduce_scatter_tensor(shard, grad_pad, op=dist.ReduceOp.SUM, group=group)
        if world > 1:
            shard.mul_(1.0 / world)
    else:
        shard.copy_(grad_pad[lo:hi])
    for k, a, b in group_pieces(slices, lo, min(hi, total)):
        adam_fn(param_pad[a:b], shard[a - lo:b - lo], m_flat[a:b], v_flat[a:b], k)
    if collective:
        dist.all_gather_into_tensor(param_pad, param_pad[lo:hi].clone(), group=group)
    grad_pad.zero_()


class DataParallelTrainStep(TrainStep):
    """TrainStep whose update is the data-parallel one: the backward writes this
    rank's gradient (gs_render_backward), then exchange_and_update runs the
    reduce-scatter, Adam on this rank's shard (gs_adam_step) and the all-gather.
    The model's parameter and gradient buffers are moved into padded storage so
    the collectives work in place. With torch.distributed initialised the
    collectives run even for one rank; without it the step is the single-GPU one.
    Densification reallocates the model's buffers: build a new step after it."""

    def __init__(self, model, max_entries, width, height, group=None, **kw):
        kw["fused_adam"] = False
        super().__init__(model, max_entries, width, height, **kw)
        self.group = group
        on = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if on else 1
        self.rank = dist.get_rank(group) if on else 0
        self.total = model.flat.numel()
        pad = padded_size(self.total, self.world)
        dev = model.flat.device
        self.param_pad = torch.zeros(pad, dtype=torch.float32, device=dev)
        self.grad_pad = torch.zeros(pad, dtype=torch.float32, device=dev)
        self.param_pad[: self.total].copy_(model.flat)
        model.attach_storage(self.param_pad[: self.total], self.grad_pad[: self.total])

    @property
    def adam_launches(self):
        lo, hi = shard_bounds(self.total, self.world, self.rank)
        return len(group_pieces(self.model.slices, lo, min(hi, self.total)))

    def update_from_grads(self):
        """Reduce-scatter, Adam on this rank's shard, all-gather."""
        m = self.model
        step = m.step_count

        def adam(p, g, mm, vv, k):
            native.adam_step(p, g, mm, vv, self.lrs[k], step, self.betas[0], self.betas[1], self.eps)

        exchange_and_update(self.grad_pad, self.param_pad, m.m_flat, m.v_flat, m.slices, self.total,
                            self.world, self.rank, adam, self.group)
