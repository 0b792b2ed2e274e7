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


def gaussian_bounds(n_pad: int, world: int, rank: int):
    """[g_lo, g_hi) of the Gaussians rank owns in the "views" exchange: equal
    ranges of whole float4 columns (multiples of 4 Gaussians), the last one
    shorter when n_pad does not split evenly."""
    per = (n_pad // 4 + world - 1) // world * 4
    lo = min(n_pad, rank * per)
    return lo, min(n_pad, lo + per)


def gather_gaussian_shards(flat, n_pad, world, rank, group=None):
    """The full planar buffer `flat` (every group's planes of n_pad Gaussians back
    to back) assembled from every rank's own Gaussians [g_lo, g_hi) of each plane:
    each rank zeroes the scalars it does not own and the buffers are summed
    (every scalar has exactly one owner, so the sum is that owner's value)."""
    collective = dist.is_available() and dist.is_initialized() and world > 1
    if not collective:
        return flat.clone()
    lo, hi = gaussian_bounds(n_pad, world, rank)
    col = torch.arange(flat.numel(), device=flat.device) % n_pad
    mine = torch.where((col >= lo) & (col < hi), flat, torch.zeros_like(flat))
    dist.all_reduce(mine, op=dist.ReduceOp.SUM, group=group)
    return mine


def gather_shards(flat, total, world, rank, group=None):
    """The full buffer of `total` floats assembled from every rank's own shard of
    `flat` (each rank's values outside its shard are ignored): the Adam moments
    of a data-parallel model, where each rank updates only its shard. A copy on
    the same device; `flat` itself is untouched."""
    collective = dist.is_available() and dist.is_initialized() and world > 1
    if not collective:
        return flat[:total].clone()
    pad = padded_size(total, world)
    lo, hi = shard_bounds(total, world, rank)
    mine = torch.zeros(hi - lo, dtype=flat.dtype, device=flat.device)
    top = min(hi, total)
    if lo < top:
        mine[: top - lo].copy_(flat[lo:top])
    out = torch.empty(pad, dtype=flat.dtype, device=flat.device)
    dist.all_gather_into_tensor(out, mine, group=group)
    return out[:total].clone()


def p2p_pieces(slices, total, world, rank, param_ptrs, grad_ptrs):
    """The gs_adam_step_reduce calls of one rank: for each parameter-group piece
    of its shard, (group, start, stop, gradient source addresses in rank order,
    addresses of the other ranks' parameter copies). Addresses are those of
    each rank's padded float32 buffer."""
    lo, hi = shard_bounds(total, world, rank)
    out = []
    for k, a, b in group_pieces(slices, lo, min(hi, total)):
        out.append((k, a, b, [g + 4 * a for g in grad_ptrs],
                    [p + 4 * a for r, p in enumerate(param_ptrs) if r != rank]))
    return out


class DataParallelTrainStep(TrainStep):
    """TrainStep whose update is the data-parallel one. With exchange="views"
    (default) each rank runs only the blend backward of its camera
    (gs_render_backward_screen); then one gs_adam_step_views launch on each rank
    reads every rank's view of the Gaussians it owns (screen records, raw screen
    sums, flags and camera, from peer memory), runs the projection backward of
    every view, averages in rank order, applies Adam and writes the updated
    parameters into every rank's buffer: no gradient buffer is written or
    exchanged. With exchange="p2p" the backward writes this rank's gradient
    (gs_render_backward), and one gs_adam_step_reduce launch per parameter
    group in this rank's shard reads every rank's gradient of the shard from
    peer memory, averages it in rank order, runs Adam and writes the updated
    shard into every rank's parameters; with exchange="nccl",
    exchange_and_update runs NCCL's reduce-scatter, gs_adam_step on the shard
    and NCCL's all-gather. All three give the same bits.

    The parameter and gradient buffers are padded so every rank's shard has
    the same size and 16-byte-aligned bounds; for "p2p" they are shared
    (gs_shared_alloc) and mapped by every other rank. With torch.distributed
    initialised the exchange runs even for one rank; without it the step is the
    single-GPU one. Densification reallocates the model's buffers: build a new
    step after it. Call close() on every rank before the step is dropped."""

    def __init__(self, model, max_entries, width, height, group=None, exchange="views", **kw):
        if exchange not in ("views", "p2p", "nccl"):
            raise ValueError("exchange must be 'views', 'p2p' or 'nccl'")
        kw["fused_adam"] = False
        super().__init__(model, max_entries, width, height, **kw)
        self.group = group
        self.exchange = exchange
        on = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if on else 1
        self.rank = dist.get_rank(group) if on else 0
        if self.world > native.MAX_RANKS:
            raise ValueError(f"at most {native.MAX_RANKS} ranks (one node)")
        self.total = model.flat.numel()
        pad = padded_size(self.total, self.world)
        dev = model.flat.device
        self._peer_maps = []
        if exchange == "views":
            self._init_views(model, on)
            return
        if exchange == "p2p":
            self._bufs = (native.SharedBuffer(pad), native.SharedBuffer(pad))
            self.param_pad, self.grad_pad = self._bufs[0].tensor, self._bufs[1].tensor
            mine = (self._bufs[0].ptr, self._bufs[1].ptr)
            if self.world > 1:
                handles = [None] * self.world
                dist.all_gather_object(handles, (self._bufs[0].handle, self._bufs[1].handle), group=group)
                ptrs = []
                for r, (hp, hg) in enumerate(handles):
                    if r == self.rank:
                        ptrs.append(mine)
                    else:
                        pair = (native.shared_open(hp), native.shared_open(hg))
                        self._peer_maps.extend(pair)
                        ptrs.append(pair)
            else:
                ptrs = [mine]
            self.param_ptrs = [p for p, _ in ptrs]
            self.grad_ptrs = [g for _, g in ptrs]
        else:
            self.param_pad = torch.zeros(pad, dtype=torch.float32, device=dev)
            self.grad_pad = torch.zeros(pad, dtype=torch.float32, device=dev)
        self.param_pad[: self.total].copy_(model.flat)
        model.attach_storage(self.param_pad[: self.total], self.grad_pad[: self.total], owner=self)
        self._flag = torch.zeros(1, dtype=torch.float32, device=dev)
        self._nccl = on and dist.get_backend(group) == "nccl"

    def _init_views(self, model, on):
        """Shared parameter buffer, this context's view buffers shared with the other
        ranks, and the views / copies of every rank."""
        self._bufs = (native.SharedBuffer(self.total),)
        self.param_pad = self._bufs[0].tensor
        self.param_pad.copy_(model.flat)
        model.attach_storage(self.param_pad, model.grad_flat, owner=self)
        self.g_lo, self.g_hi = gaussian_bounds(model.n_pad, self.world, self.rank)
        my_view = self.ctx.view()
        fields = native.GsView.FIELDS
        views = [None] * self.world
        views[self.rank] = my_view
        self.copies = []
        if self.world > 1:
            mine = (self._bufs[0].handle, [native.shared_handle(getattr(my_view, f)) for f in fields])
            handles = [None] * self.world
            dist.all_gather_object(handles, mine, group=self.group)
            for r, (hp, hv) in enumerate(handles):
                if r == self.rank:
                    continue
                ptrs = [native.shared_open(h) for h in hv]
                self._peer_maps.extend(ptrs)
                views[r] = native.GsView(*ptrs)
                base = native.shared_open(hp)
                self._peer_maps.append(base)
                self.copies.append(native.GsGrads(*[base + 4 * model.slices[k].start for k in GROUP_NAMES]))
        self.views = views
        self._flag = torch.zeros(1, dtype=torch.float32, device=model.flat.device)
        self._nccl = on and dist.get_backend(self.group) == "nccl"

    def backward_and_update(self, cs, T, nc, dimg):
        """The "views" exchange: this rank's blend backward, then the update of its
        Gaussians from every rank's view (the other exchanges: TrainStep's path)."""
        if self.exchange != "views":
            return super().backward_and_update(cs, T, nc, dimg)
        m = self.model
        m.step_count += 1
        self.ctx.render_backward_screen(m.params_struct(), cs, T, nc, dimg)
        self._barrier()  # every rank's view is complete
        em, ev = m.moments_structs()
        self.ctx.adam_step_views(m.params_struct(), self.views, self.g_lo, self.g_hi, self.copies, em, ev,
                                 [self.lrs[k] for k in GROUP_NAMES], m.step_count, beta1=self.betas[0],
                                 beta2=self.betas[1], eps=self.eps)
        self._barrier()  # every rank's copies have landed

    def _barrier(self):
        """Every rank's work enqueued so far is complete before anything enqueued after
        it runs: a one-float all-reduce on the stream (NCCL), or a device
        synchronise plus a host barrier (other backends)."""
        if self.world == 1:
            return
        if self._nccl:
            dist.all_reduce(self._flag, group=self.group)
        else:
            torch.cuda.synchronize()
            dist.barrier(group=self.group)

    @property
    def adam_launches(self):
        if self.exchange == "views":
            return 1
        lo, hi = shard_bounds(self.total, self.world, self.rank)
        return len(group_pieces(self.model.slices, lo, min(hi, self.total)))

    def update_from_grads(self):
        """The exchange and the Adam step of this rank's shard."""
        m = self.model
        step = m.step_count
        b1, b2 = self.betas
        if self.exchange == "nccl":
            def adam(p, g, mm, vv, k):
                native.adam_step(p, g, mm, vv, self.lrs[k], step, b1, b2, self.eps)

            exchange_and_update(self.grad_pad, self.param_pad, m.m_flat, m.v_flat, m.slices, self.total,
                                self.world, self.rank, adam, self.group)
            return
        self._barrier()  # every rank's gradient is complete
        one = self.world == 1
        for k, a, b, gsrc, copies in p2p_pieces(m.slices, self.total, self.world, self.rank,
                                                self.param_ptrs, self.grad_ptrs):
            native.adam_step_reduce(self.param_pad[a:b], m.m_flat[a:b], m.v_flat[a:b], gsrc, copies,
                                    self.lrs[k], step, grad_scale=1.0 / self.world, zero_grads=one,
                                    beta1=b1, beta2=b2, eps=self.eps)
        if not one:
            self._barrier()  # every shard is read and every copy written
            self.grad_pad.zero_()

    def state_dict(self) -> dict:
        """The model's training state with the Adam moments of every rank's shard
        gathered (collective: every rank calls it; every rank gets the full state)."""
        m = self.model
        if self.exchange == "views":
            mf = gather_gaussian_shards(m.m_flat, m.n_pad, self.world, self.rank, self.group)
            vf = gather_gaussian_shards(m.v_flat, m.n_pad, self.world, self.rank, self.group)
        else:
            mf = gather_shards(m.m_flat, self.total, self.world, self.rank, self.group)
            vf = gather_shards(m.v_flat, self.total, self.world, self.rank, self.group)
        return m.state_dict(m_flat=mf, v_flat=vf)

    def load_state_dict(self, state: dict):
        """Restores a full state (as state_dict gives) on this rank: the parameters into
        the shared buffers, the moments of every shard, the step count. The state must
        have this step's sizes."""
        m = self.model
        if int(state["n_pad"]) != m.n_pad:
            raise ValueError("the state has another size: build a new step for it")
        m.load_state_dict(state)

    def close(self):
        """Unmaps the other ranks' buffers; collective when there are several ranks
        (no rank frees its buffers while another still maps them)."""
        if self._peer_maps:
            self._barrier()
            for p in self._peer_maps:
                native.shared_close(p)
            self._peer_maps = []
            self._barrier()
