"""Saving and restoring the training state (parameters, Adam moments, sizes,
step count) of a GaussianModel; the buffers live wherever the model does, so
this runs on the host."""
import io

import torch

from gaussian_splatting_differentiable_rasteriser_b200 import model, scenes


def test_state_round_trips_through_torch_save():
    a = model.GaussianModel(scenes.tiny(), device="cpu")
    a.m_flat.normal_()
    a.v_flat.uniform_()
    a.step_count = 17
    a.active_degree = 0
    buf = io.BytesIO()
    torch.save(a.state_dict(), buf)
    buf.seek(0)
    b = model.GaussianModel(scenes.tiny(seed=1), device="cpu")
    b.load_state_dict(torch.load(buf))
    assert torch.equal(a.flat, b.flat) and torch.equal(a.m_flat, b.m_flat) and torch.equal(a.v_flat, b.v_flat)
    assert (b.n, b.n_pad, b.step_count, b.active_degree) == (a.n, a.n_pad, 17, 0)
    for k in scenes.GROUP_NAMES:  # the group views point into the restored buffers
        assert torch.equal(a.params[k], b.params[k])


def test_state_of_another_sh_degree_is_refused():
    import pytest
    a = model.GaussianModel(scenes.tiny(), device="cpu")
    b = model.GaussianModel(scenes.small(), device="cpu")
    with pytest.raises(ValueError):
        b.load_state_dict(a.state_dict())
