import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def to64(t):
    """bf16/fp32 torch tensor -> float64 numpy (exact widening)."""
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.fixture
def rng():
    return np.random.default_rng(12345)
