import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")


@pytest.fixture(scope="session")
def cuda_available():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="session")
def colimoe():
    """The CUDA library, built in-tree if stale (needs nvcc only, no GPU)."""
    from int4_routed_expert_gemv_b200 import build, binding
    build.build()
    binding.lib()
    return binding
