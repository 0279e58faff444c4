import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running parity case")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA branch-attention library, loaded through its C-ABI binding."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_draft_branch_b200 as ba
    return ba
