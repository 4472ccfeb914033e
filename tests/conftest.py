import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_lib():
    """The loaded CUDA library; GPU tests fail loudly when it is missing."""
    from head_split_kv_decode_b200 import binding
    if not has_gpu():
        pytest.fail("gpu test selected but no CUDA device is visible")
    return binding.lib()
