import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def lib():
    """The CUDA library through its C-ABI binding; fails loudly if missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fine_grained_fp8_sigmoid_b200 import _lib
    return _lib.load()
