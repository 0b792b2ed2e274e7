"""Device-resident Gaussian parameters and one training step through the C ABI.

Holds the parameters, their gradients and the two Adam moments as four flat
float32 buffers with one planar view per group (so each group's start is
16-byte aligned and Adam streams it with float4 accesses), and sequences the
five entry points of one iteration: preprocess -> render_forward ->
loss_l1_dssim -> render_backward -> adam_step (once per group, each with its
own learning rate, as "Differentiable rasterisation" (splat-report), section
"From a pixel error back to a quaternion", describes).
"""
from __future__ import annotations

import torch

from . import native
from .scenes import GROUP_NAMES


def group_shapes(n_pad: int, sh_degree: int) -> dict:
    K = (sh_degree + 1) ** 2
    return {"means": (3, n_pad), "log_scales": (3, n_pad), "quats": (4, n_pad),
            "opacity_logits": (n_pad,), "sh": (3, K, n_pad)}


class GaussianModel:
    def __init__(self, scene, device="cuda", active_degree=None):
        self.n, self.sh_degree = scene.n, scene.sh_degree
        self.active_degree = scene.sh_degree if active_degree is None else active_degree
        self.device = device
        # set while a data-parallel step owns the parameter and gradient storage
        self.storage_owner = None
        self._alloc(scene.n_pad)
        self.load(scene)
        self.step_count = 0

    def _alloc(self, n_pad):
        """Fresh flat buffers (parameters uninitialised, the rest zero) for n_pad slots."""
        self.n_pad = n_pad
        shapes = group_shapes(n_pad, self.sh_degree)
        sizes = {k: int(torch.Size(s).numel()) for k, s in shapes.items()}
        total = sum(sizes.values())
        dev = self.device
        self.flat = torch.empty(total, dtype=torch.float32, device=dev)
        self.grad_flat = torch.zeros(total, dtype=torch.float32, device=dev)
        self.m_flat = torch.zeros(total, dtype=torch.float32, device=dev)
        self.v_flat = torch.zeros(total, dtype=torch.float32, device=dev)
        self.params, self.grads, self.m, self.v, self.slices = {}, {}, {}, {}, {}
        off = 0
        for k in GROUP_NAMES:
            sl = slice(off, off + sizes[k])
            self.slices[k] = sl
            self.params[k] = self.flat[sl].view(shapes[k])
            self.grads[k] = self.grad_flat[sl].view(shapes[k])
            self.m[k] = self.m_flat[sl].view(shapes[k])
            self.v[k] = self.v_flat[sl].view(shapes[k])
            off += sizes[k]

    def attach_storage(self, flat, grad_flat, owner=None):
        """Moves the parameters and gradients into the given flat buffers (same size;
        the current parameters must already be in `flat`) and rebuilds the group views.
        `owner` (the data-parallel step that made the buffers) is recorded: while it is
        set, state_dict() refuses (the owner's state_dict gathers the moments of every
        rank) and load_state_dict() refuses a change of size."""
        assert flat.numel() == self.flat.numel() and grad_flat.numel() == self.grad_flat.numel()
        self.storage_owner = owner
        self.flat, self.grad_flat = flat, grad_flat
        shapes = group_shapes(self.n_pad, self.sh_degree)
        for k in GROUP_NAMES:
            sl = self.slices[k]
            self.params[k] = self.flat[sl].view(shapes[k])
            self.grads[k] = self.grad_flat[sl].view(shapes[k])

    def relocate(self, ctx, normals, dead_opacity=0.02, donor_opacity=0.4):
        """Recycles dead Gaussians onto the largest donors in place (gs_relocate);
        normals: [pairs, 3] float32 N(0, 1) draws on the device, one row per pair
        at most. Returns the number of pairs made."""
        em, ev = self.moments_structs()
        return ctx.relocate(self._struct(self.params), em, ev, self.n, self.n_pad, self.sh_degree, normals,
                            normals.shape[0], dead_opacity, donor_opacity)

    def densify(self, ctx, grad_accum, view_count, normals, grad_threshold, scale_threshold,
                min_opacity, capacity=None):
        """One gs_densify pass into new buffers of `capacity` slots (default: room
        for every Gaussian to split); the model then holds the new set, its
        moments and zeroed gradients. Returns the new count."""
        p_in, (m_in, v_in) = self.params_struct(), self.moments_structs()
        keep = (self.flat, self.m_flat, self.v_flat, self.grad_flat)  # alive until the call returns
        cap = capacity if capacity is not None else max(4, (2 * self.n + 3) // 4 * 4)
        old_params, old_m, old_v = self.params, self.m, self.v
        self._alloc(cap)
        self.flat.zero_()
        out, (m_out, v_out) = self._struct(self.params), self.moments_structs()
        n_out = ctx.densify(p_in, m_in, v_in, grad_accum, view_count, normals, grad_threshold,
                            scale_threshold, min_opacity, out, m_out, v_out, cap)
        del keep, old_params, old_m, old_v
        self.n = n_out
        return n_out

    def load(self, scene):
        for k in GROUP_NAMES:
            self.params[k].copy_(torch.from_numpy(getattr(scene, k)).to(torch.float32))

    def state_dict(self, m_flat=None, v_flat=None) -> dict:
        """Training state for torch.save: parameters and both Adam moments (flat,
        planar group layout, copied to the host), sizes, degrees and the step count.
        The gradient buffer is not saved: it is zero between iterations. Refused while
        a data-parallel step owns the storage, since each rank then holds the moments
        of its own shard only: save through that step's state_dict(), which passes the
        gathered moments here."""
        if self.storage_owner is not None and m_flat is None:
            raise RuntimeError("a data-parallel step owns this model's storage: save with its state_dict()")
        m_flat = self.m_flat if m_flat is None else m_flat
        v_flat = self.v_flat if v_flat is None else v_flat
        return {"flat": self.flat.detach().cpu().clone(), "m_flat": m_flat.detach().cpu().clone(),
                "v_flat": v_flat.detach().cpu().clone(), "n": self.n, "n_pad": self.n_pad,
                "sh_degree": self.sh_degree, "active_degree": self.active_degree,
                "step_count": self.step_count}

    def load_state_dict(self, state: dict):
        """Restores a state_dict (reallocating if the padded size differs; refused
        while a data-parallel step owns the storage, whose buffers keep their size:
        build a new step for another size)."""
        if state["sh_degree"] != self.sh_degree:
            raise ValueError("the state was saved with another SH degree")
        n, n_pad = int(state["n"]), int(state["n_pad"])
        if not 0 <= n <= n_pad or n_pad % 4:
            raise ValueError("the state's sizes are inconsistent (need 0 <= n <= n_pad, n_pad % 4 == 0)")
        total = sum(int(torch.Size(s).numel()) for s in group_shapes(n_pad, self.sh_degree).values())
        for k in ("flat", "m_flat", "v_flat"):
            if state[k].numel() != total:
                raise ValueError(f"the state's {k} holds {state[k].numel()} floats, its sizes need {total}")
        if n_pad != self.n_pad:
            if self.storage_owner is not None:
                raise RuntimeError("a data-parallel step owns this model's storage: its size cannot change")
            self._alloc(n_pad)
        self.flat.copy_(state["flat"])
        self.m_flat.copy_(state["m_flat"])
        self.v_flat.copy_(state["v_flat"])
        self.grad_flat.zero_()
        self.n = state["n"]
        self.active_degree = state["active_degree"]
        self.step_count = state["step_count"]

    def params_struct(self) -> native.GsParams:
        p = native.GsParams()
        for k in GROUP_NAMES:
            setattr(p, k, self.params[k].data_ptr())
        p.n, p.n_pad = self.n, self.n_pad
        p.sh_degree, p.active_degree = self.sh_degree, self.active_degree
        return p

    def _struct(self, tensors) -> native.GsGrads:
        g = native.GsGrads()
        for k in GROUP_NAMES:
            setattr(g, k, tensors[k].data_ptr())
        return g

    def grads_struct(self) -> native.GsGrads:
        return self._struct(self.grads)

    def moments_structs(self):
        return self._struct(self.m), self._struct(self.v)


DEFAULT_LR = {k: 1e-3 for k in GROUP_NAMES}


def sh_degree_at(step: int, every: int, max_degree: int) -> int:
    """SH bands unlocked before iteration `step` (0-based) when one more degree is
    switched on every `every` iterations ("How a computer rebuilds a real place ...
    Gaussian Splats", section "Spherical harmonics: color that changes with viewing
    angle": degree 0 first, one degree about every 1000 steps)."""
    return min(max_degree, step // every)


class TrainStep:
    """Buffers and the call sequence of one iteration for images up to width x height."""

    def __init__(self, model: GaussianModel, max_entries: int, width: int, height: int, lrs=None,
                 lam=0.2, betas=(0.9, 0.999), eps=1e-8, device="cuda", fused_adam=True,
                 opacity_rect=False, deterministic=False, loss="l1_dssim", sh_ramp_every=None,
                 mip_comp=False):
        self.model = model
        # None: the model's active degree stays as set; otherwise it follows sh_degree_at
        self.sh_ramp_every = sh_ramp_every
        self.fused_adam = fused_adam
        if loss not in ("l1_dssim", "charbonnier"):
            raise ValueError("loss must be 'l1_dssim' or 'charbonnier'")
        self.loss_kind = loss
        # per-photo exposure of the Charbonnier loss (identity by default)
        self.gain, self.bias = [1.0, 1.0, 1.0], [0.0, 0.0, 0.0]
        self.ctx = native.Context(model.n_pad, max_entries, width, height)
        if opacity_rect:
            self.ctx.set_option(native.GS_OPTION_OPACITY_RECT, 1)
        if deterministic:
            self.ctx.set_option(native.GS_OPTION_DETERMINISTIC, 1)
        if mip_comp:  # opacities times the Mip-Splatting compensation factor
            self.ctx.set_option(native.GS_OPTION_MIP_COMPENSATION, 1)
        self.lrs = dict(DEFAULT_LR if lrs is None else lrs)
        self.lam, self.betas, self.eps = lam, betas, eps
        self.image = torch.empty((3, height, width), dtype=torch.float32, device=device)
        self.final_T = torch.empty((height, width), dtype=torch.float32, device=device)
        self.n_contrib = torch.empty((height, width), dtype=torch.int32, device=device)
        self.dimage = torch.empty((3, height, width), dtype=torch.float32, device=device)
        # {loss, L1, SSIM}, or for the Charbonnier loss {loss, dL/dgain[3], dL/dbias[3]}
        self.loss = torch.zeros(7, dtype=torch.float64, device=device)
        self.last_entries = 0

    def forward(self, cam_struct, H, W):
        p = self.model.params_struct()
        self.ctx.preprocess(p, cam_struct)
        img, T, nc = self.image[:, :H, :W], self.final_T[:H, :W], self.n_contrib[:H, :W]
        if H != self.image.shape[1] or W != self.image.shape[2]:
            img = torch.empty((3, H, W), dtype=torch.float32, device=self.image.device)
            T = torch.empty((H, W), dtype=torch.float32, device=self.image.device)
            nc = torch.empty((H, W), dtype=torch.int32, device=self.image.device)
        self.last_entries = self.ctx.render_forward(cam_struct, img, T, nc)
        return img, T, nc

    def __call__(self, cam, target):
        """One iteration against `target` ([3, H, W] float32 on the device)."""
        if self.sh_ramp_every:
            m = self.model
            m.active_degree = sh_degree_at(m.step_count, self.sh_ramp_every, m.sh_degree)
        cs = native.camera_struct(cam)
        H, W = cam.height, cam.width
        img, T, nc = self.forward(cs, H, W)
        dimg = self.dimage if img.shape == self.dimage.shape else torch.empty_like(img)
        self.compute_loss(img, target, dimg)
        self.backward_and_update(cs, T, nc, dimg)
        return self.loss

    def compute_loss(self, img, target, dimg):
        """The configured loss of `img` against `target`, its gradient into dimg."""
        if self.loss_kind == "charbonnier":
            self.ctx.loss_charbonnier(img, target, self.gain, self.bias, self.loss, dimg)
        else:
            self.ctx.loss_l1_dssim(img, target, self.lam, self.loss, dimg)

    def backward_and_update(self, cs, T, nc, dimg):
        """Backward of the last forward plus the Adam step of every group: one fused
        pass over the parameters, or gs_render_backward then gs_adam_step per group."""
        m = self.model
        m.step_count += 1
        if self.fused_adam:
            # one view per step: no accumulated gradient, so no gradient buffer traffic
            em, ev = m.moments_structs()
            self.ctx.render_backward_adam(m.params_struct(), cs, T, nc, dimg, None, em, ev,
                                          [self.lrs[k] for k in GROUP_NAMES], m.step_count,
                                          self.betas[0], self.betas[1], self.eps)
            return
        self.ctx.render_backward(m.params_struct(), cs, T, nc, dimg, m.grads_struct())
        self.update_from_grads()

    # gs_adam_step launches of one update_from_grads call
    adam_launches = len(GROUP_NAMES)

    def update_from_grads(self):
        """Adam on every group from the gradient buffer (which it zeroes), at the
        model's current step count."""
        m = self.model
        for k in GROUP_NAMES:
            native.adam_step(m.params[k], m.grads[k], m.m[k], m.v[k], self.lrs[k], m.step_count,
                             self.betas[0], self.betas[1], self.eps)
