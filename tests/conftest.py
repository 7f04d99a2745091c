import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def native():
    """The built libpagedkv (compiled on first use; nvcc cross-compiles sm_100a
    without a GPU)."""
    from paged_kv_cache_406_b200 import build
    build.build()
    from paged_kv_cache_406_b200 import _native
    return _native.lib()


def cuda_ok() -> bool:
    import torch
    return torch.cuda.is_available()
