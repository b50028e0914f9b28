import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")
    config.addinivalue_line("markers", "slow: full-size parity case")


@pytest.fixture(scope="session")
def lib():
    """The product library (CUDA path). Only GPU tests use it."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_w8a8_linear_b200 as f

    return f
