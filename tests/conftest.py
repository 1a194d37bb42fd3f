import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle
    _oracle.build()
    return _oracle


@pytest.fixture(scope="session")
def rfq():
    """The CUDA path's Python binding, with the library loaded (GPU tests only)."""
    if not cuda_available():
        pytest.fail("GPU test collected on a host without CUDA")
    import block_scaled_gemm_rfq_b200 as _rfq
    _rfq.load_library()
    return _rfq
