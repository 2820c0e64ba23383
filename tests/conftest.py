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


# parity bar for bf16 outputs against the fp64 oracle: max |err| <= 2e-2 and
# relative L2 error <= 5e-3 (the layer's stated tolerance)
MAX_ABS = 2e-2
REL_L2 = 5e-3


def errors(got, ref):
    """(max |got - ref|, ||got - ref|| / ||ref||) with got any array-like of bf16/float."""
    import numpy as np
    import torch
    if isinstance(got, torch.Tensor):
        got = got.detach().to("cpu", torch.float64).numpy()
    got = np.asarray(got, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    diff = got - ref
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30))


def assert_parity(got, ref, what=""):
    mx, rl = errors(got, ref)
    assert mx <= MAX_ABS and rl <= REL_L2, f"{what}: max|err| {mx:.3e}, rel-L2 {rl:.3e}"
    return mx, rl


def need_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
