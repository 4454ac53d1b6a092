import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


def cuda_ok() -> bool:
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="session")
def rkv():
    """The CUDA library binding; GPU tests fail loudly if it is missing."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import retention_scored_kv_b200 as rkv_mod
    rkv_mod.load()
    return rkv_mod
