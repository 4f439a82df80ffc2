import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def svo():
    """The C oracle (built on first use)."""
    import oracle
    oracle.lib()
    return oracle


def _cuda_ok():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def sv():
    """The CUDA library's Python binding; GPU tests only."""
    if not _cuda_ok():
        pytest.skip("no CUDA device")
    import speculative_decoding_verification_lse_b200 as sv
    sv.load()
    return sv
