import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def built_library():
    """Path of libdora.so, building it in-tree with nvcc if it is missing."""
    from dora_adapter_factored_b200 import build as _build
    path = _build.library_path()
    if not os.path.exists(path) or _build.is_stale():
        _build.build()
    return path


@pytest.fixture(scope="session")
def built_debug_library():
    """Path of libdora_debug.so (the DORA_DEBUG build), building it if needed."""
    from dora_adapter_factored_b200 import build as _build
    path = _build.library_path(debug=True)
    if not os.path.exists(path) or _build.is_stale(debug=True):
        _build.build(debug=True)
    return path
