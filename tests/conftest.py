import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def has_cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def metis():
    """The CUDA library's Python binding, on a machine with a GPU only (never a fallback)."""
    if not has_cuda():
        pytest.fail("GPU test collected on a machine without CUDA; run with -m 'not gpu'")
    from moe_gemm_token_b200 import metis as m
    m.load()
    return m
