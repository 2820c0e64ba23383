"""Output sconv (window-4 short convolution on the attention output) on the
GPU against the oracle's sconv, plus streaming through the state."""
import numpy as np
import pytest
import torch

from conftest import assert_append_close, need_gpu, u16
import relative_bias_sliding_b200 as ink

pytestmark = pytest.mark.gpu


def _inputs(B, T, C, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, T, C), generator=g).to(torch.bfloat16)
    w = torch.randn((C, 4), generator=g) * 0.5
    state = torch.randn((B, 3, C), generator=g).to(torch.bfloat16)
    return x, w, state


@pytest.mark.parametrize("T", [1, 2, 3, 31, 32, 33, 100, 1000])
@pytest.mark.parametrize("with_state", [False, True])
def test_sconv_out_matches_oracle(oracle_mod, T, with_state):
    need_gpu()
    B, C = 3, 1024
    x, w, state = _inputs(B, T, C, seed=T + 7 * with_state)
    st = state.cuda() if with_state else None
    y = ink.sconv_out(x.cuda(), w.cuda(), st)
    torch.cuda.synchronize()
    ref = oracle_mod.sconv(u16(x), w.numpy(), u16(state) if with_state else None)
    frac = assert_append_close(u16(y), ref)
    assert frac < 2e-3
    if with_state:
        # the new state is the last 3 raw rows of (old state, x): exact
        full = torch.cat([state, x], dim=1)
        assert torch.equal(st.cpu(), full[:, -3:])


def test_sconv_out_streaming_equals_one_shot():
    """Chunks of 1, 5, 64, 930 tokens through the state give the one-shot output."""
    need_gpu()
    B, T, C = 2, 1000, 8192   # C = 64 query heads x 128
    x, w, _ = _inputs(B, T, C, seed=3)
    xd, wd = x.cuda(), w.cuda()
    one = ink.sconv_out(xd, wd, torch.zeros((B, 3, C), dtype=torch.bfloat16, device="cuda"))
    st = torch.zeros((B, 3, C), dtype=torch.bfloat16, device="cuda")
    parts, t = [], 0
    for n in (1, 5, 64, 930):
        parts.append(ink.sconv_out(xd[:, t:t + n].contiguous(), wd, st))
        t += n
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), one)
    # zero history is the same as a zero state
    assert torch.equal(ink.sconv_out(xd, wd), one)


def test_sconv_out_rejects_overlap_and_bad_channels():
    need_gpu()
    x, w, _ = _inputs(1, 16, 64, seed=1)
    xd = x.cuda()
    with pytest.raises(ink.InklingError):
        ink.sconv_out(xd, w.cuda(), out=xd)
    with pytest.raises(ink.InklingError):   # channels must be a multiple of 8
        ink.sconv_out(xd[:, :, :60].contiguous(), w[:60].contiguous().cuda())
