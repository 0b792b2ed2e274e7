"""The allocation-free loss entry point (for callers that cannot call cudaMalloc
where they need the loss: a host whose own allocator owns the GPU's memory, or a
real-time loop whose memory is fixed after start-up) must give the same loss and
image gradient as the context-based entry point. It runs the same kernel on the
same inputs with a fixed-order reduction, so both must agree bit for bit.

Called through the C ABI directly. Collected last (file name) so that a run that
stops at the first failure has already run every other test; it passes both on
its own in a fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("shape", [(256, 256), (70, 33)])
def test_noalloc_loss_matches_context_loss_twice(shape):
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    assert torch.cuda.is_available(), "needs a CUDA device"
    L = native.load()
    H, W = shape
    rng = np.random.default_rng(H + W)
    x = torch.from_numpy(rng.uniform(0, 1, (3, H, W)).astype(np.float32)).cuda()
    y = torch.from_numpy(rng.uniform(0, 1, (3, H, W)).astype(np.float32)).cuda()
    ctx = native.Context(16, 16, W, H)
    ref_loss = torch.zeros(3, dtype=torch.float64, device="cuda")
    ref_d = torch.empty((3, H, W), device="cuda")
    ctx.loss_l1_dssim(x, y, 0.2, ref_loss, ref_d)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):  # the shared scratch must be reusable call after call
        loss = torch.full((3,), -1.0, dtype=torch.float64, device="cuda")
        d = torch.full((3, H, W), float("nan"), device="cuda")
        st = L.gs_loss_l1_dssim_noalloc(_ptr(x), _ptr(y), H, W, ctypes.c_float(0.2), _ptr(loss), _ptr(d),
                                        stream)
        assert st == native.GS_OK
        torch.cuda.synchronize()
        np.testing.assert_array_equal(loss.cpu().numpy(), ref_loss.cpu().numpy())
        np.testing.assert_array_equal(d.cpu().numpy(), ref_d.cpu().numpy())


def test_noalloc_loss_rejects_images_beyond_its_scratch():
    import __graft_entry__
    __graft_entry__.build()
    from gaussian_splatting_differentiable_rasteriser_b200 import native
    L = native.load()
    dummy = torch.zeros(4, device="cuda")
    loss = torch.zeros(3, dtype=torch.float64, device="cuda")
    st = L.gs_loss_l1_dssim_noalloc(_ptr(dummy), _ptr(dummy), 4097, 16, ctypes.c_float(0.2), _ptr(loss),
                                    None, None)
    assert st == native.GS_ERR_CAPACITY
