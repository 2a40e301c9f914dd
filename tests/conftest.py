import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(scope="session", autouse=True)
def _library_built():
    """Build libmoe_mx.so (and nothing else) if it is missing or older than its sources, so
    that the tests always load the library built from the sources they test."""
    from block_scaled_moe_softmax_b200 import build as lib_build
    lib_build.build()


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()
