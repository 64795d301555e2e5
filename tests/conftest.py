import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def _has_gpu() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_ok():
    if not _has_gpu():
        pytest.skip("no CUDA device")
    return True


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Compile libnvfp4.so (nvcc, sm_100a) if a source changed; cheap otherwise."""
    from nvfp4_w4a4_gemm_quantize_b200 import build
    build.build()
