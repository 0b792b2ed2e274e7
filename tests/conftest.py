import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built extension")


def golden(name: str) -> dict:
    """Parses a `key = value` fixture under tests/golden; numeric values become
    floats or float arrays, anything else stays a string."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (s.strip() for s in line.split("=", 1))
            parts = v.split()
            try:
                nums = [float(p) for p in parts]
                out[k] = nums[0] if len(nums) == 1 else np.array(nums)
            except ValueError:
                out[k] = v
    return out


@pytest.fixture
def gold():
    return golden
