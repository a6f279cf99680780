import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: larger CPU cases")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def sbn_lib():
    """libsbn.so, built in-tree if missing or stale (nvcc cross-compiles here)."""
    from sparse_linear_layers_fwd_b200 import build, sbn
    build.build()
    return sbn.lib()


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True
