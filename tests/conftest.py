import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library; GPU tests fail loudly when it is missing."""
    import torch
    from exact_tiled_attention_45_b200 import binding
    assert torch.cuda.is_available(), "gpu-marked test needs a CUDA device"
    return binding.load()
