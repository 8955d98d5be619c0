import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes of CPU oracle time)")


@pytest.fixture(scope="session")
def lib():
    """The CUDA library through its ctypes binding; GPU tests only."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_absorption_b200 import build
    build.build()
    from kv_cache_absorption_b200 import ispa
    ispa._load()
    return ispa
