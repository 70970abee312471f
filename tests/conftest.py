import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large oracle work (minutes)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The loaded CUDA library (fails loudly if it is missing or no GPU is present)."""
    import torch

    if not torch.cuda.is_available():
        pytest.fail("gpu test collected on a machine without CUDA")
    import sparse_linear_attention_pool_b200 as sla

    sla.load()
    return sla
