import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libcalibq")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_device():
    if not gpu_available():
        pytest.skip("no CUDA device")
    return "cuda:0"


@pytest.fixture
def row_kernel(cuda_device):
    """Force the one-CTA-per-row 1-bit decode kernel for one test (it takes
    n <= 8192), then hand the choice back to the environment / estimate."""
    from decode_attention_cq_b200 import calibq as cq

    cq.cq_set_decode_kernel(cq.KERNEL_ROW)
    yield cuda_device
    cq.cq_set_decode_kernel(cq.KERNEL_ENV)


@pytest.fixture
def pipe_kernel(cuda_device):
    """Force the persistent tcgen05 1-bit decode kernel (plain decodes with
    n <= 8192) for one test, then hand the choice back."""
    from decode_attention_cq_b200 import calibq as cq

    cq.cq_set_decode_kernel(cq.KERNEL_PIPE)
    yield cuda_device
    cq.cq_set_decode_kernel(cq.KERNEL_ENV)
