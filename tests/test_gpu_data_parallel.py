"""The data-parallel step on the GPU with a one-rank NCCL group: the
reduce-scatter, the sharded Adam and the all-gather run for real, and with the
fixed-point (order-independent) gradient sums the result is bitwise the
single-GPU step's (gs_render_backward, then gs_adam_step per group)."""
import os
import socket

import numpy as np
import pytest

from gaussian_splatting_differentiable_rasteriser_b200 import scenes

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_step_equals_the_single_gpu_step():
    import datetime

    import torch.distributed as dist

    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import model, native
    from gaussian_splatting_differentiable_rasteriser_b200.data_parallel import DataParallelTrainStep
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    native.load()
    scene = scenes.small()
    cam = scene.cameras[0]
    target = torch.from_numpy(scenes.uniform_image(cam.height, cam.width, seed=3)).cuda()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        ma, mb = model.GaussianModel(scene), model.GaussianModel(scene)
        cap = 1 << 20
        a = DataParallelTrainStep(ma, cap, cam.width, cam.height, deterministic=True)
        b = model.TrainStep(mb, cap, cam.width, cam.height, fused_adam=False, deterministic=True)
        assert a.world == 1 and a.adam_launches == len(scenes.GROUP_NAMES)
        for _ in range(3):
            la, lb = a(cam, target), b(cam, target)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(la.cpu().numpy(), lb.cpu().numpy())
        assert torch.equal(ma.flat, mb.flat) and torch.equal(ma.m_flat, mb.m_flat)
        assert torch.equal(ma.v_flat, mb.v_flat)
        assert not a.grad_pad.any() and not a.param_pad[ma.flat.numel():].any()
        # the parameters moved: the step is not a no-op
        assert not torch.equal(ma.flat, model.GaussianModel(scene).flat)
    finally:
        dist.destroy_process_group()
