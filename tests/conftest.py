import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large parity case")


def u16(t):
    """torch bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
