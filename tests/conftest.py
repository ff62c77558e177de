import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a); parity tests "
                   "of the CUDA path against the oracle")


@pytest.fixture(scope="session")
def cuda_lib():
    """The product library, loaded on a GPU machine; the tests that use it are
    marked gpu."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import quantized_matmul_02_b200 as qmm
    return qmm
