"""The SH-degree ramp of the training loop ("How a computer rebuilds a real
place ... Gaussian Splats", section "Spherical harmonics: color that changes
with viewing angle": bands unlocked one degree at a time, about every 1000
steps, inactive bands unused and without gradient)."""
from gaussian_splatting_differentiable_rasteriser_b200.model import sh_degree_at


def test_one_more_degree_every_period_up_to_the_stored_degree():
    assert [sh_degree_at(s, 1000, 3) for s in (0, 999, 1000, 1999, 2000, 3000, 10_000)] == [0, 0, 1, 1, 2, 3, 3]
    assert all(sh_degree_at(s, 7, 1) <= 1 for s in range(100))
    assert sh_degree_at(5, 1, 0) == 0
