"""The decode entry point for callers that cannot allocate device memory.

inkling_attn_decode_static keeps its split partials in an array the library
owns, so a caller that can only pass inputs and outputs (no workspace) still
gets the split-KV decode.  Called here through the C ABI, twice in a row (the
array keeps the previous call's contents), and compared with
inkling_attn_decode given a workspace.  This file is collected last so that a
failure here leaves every other test already run."""
import ctypes

import pytest
import torch

from conftest import MAX_ABS, REL_L2, assert_parity, errors, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200 import binding
from relative_bias_sliding_b200.inputs import WORKLOADS, make_decode, scaled

pytestmark = pytest.mark.gpu


def _params(t, window, out, num_splits):
    return binding._decode_params(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                  t["seq_lens"], t["bias"], window, out, None, None, num_splits)


@pytest.mark.parametrize("num_splits", [0, 4])
def test_static_scratch_decode_matches_workspace_decode(num_splits):
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=12, L_min=100, L_max=20000, window=4096)
    t = make_decode(spec, device="cuda")
    ref = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                          t["bias"], window=spec.window, num_splits=num_splits)
    lib = binding.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full_like(t["q"], float("nan"))
        p = _params(t, spec.window, out, num_splits)
        assert lib.inkling_attn_decode_static(ctypes.byref(p), stream) == 0, \
            lib.inkling_last_error().decode()
        torch.cuda.synchronize()
        mx, rl = errors(out.float(), ref.float().cpu().numpy())
        assert mx <= MAX_ABS and rl <= REL_L2, f"call {call}: max {mx:.3e} rel {rl:.3e}"
        if num_splits:
            # same split count, same kernels: identical results
            assert torch.equal(out, ref)


def test_static_scratch_rejects_explicit_splits_that_do_not_fit():
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=64, L_min=1000, L_max=2000, window=0)
    t = make_decode(spec, device="cuda")
    out = torch.empty_like(t["q"])
    # 64 seqs x 64 heads x 1024 splits x 520 B = 2.2 GB of partials > 8 MiB
    p = _params(t, 0, out, 1024)
    lib = binding.load_library()
    rc = lib.inkling_attn_decode_static(ctypes.byref(p), None)
    assert rc == binding.INKLING_ERR_INVALID
    assert b"static scratch" in lib.inkling_last_error()


def _static_c(t, window, out, num_splits, status=None):
    """One inkling_attn_decode_static call through the C ABI on the current stream."""
    lib = binding.load_library()
    p = binding._decode_params(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                               t["seq_lens"], t["bias"], window, out, None, status, num_splits)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.inkling_attn_decode_static(ctypes.byref(p), stream)
    assert rc == 0, lib.inkling_last_error().decode()


@pytest.mark.parametrize("window", [0, 4096])
def test_static_scratch_decode_matches_oracle(oracle_mod, window):
    """Two calls in a row, each compared with the fp64 oracle on every
    (sequence, head) pair; few sequences, so the split count is above one and
    the partials really pass through the library's array."""
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=6, L_min=300, L_max=30000, window=window,
                  seed=21)
    t = make_decode(spec, device="cuda")
    assert ink.decode_num_splits(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                 t["seq_lens"], t["bias"], window=window) > 1
    host = {k: v.cpu() for k, v in t.items()}
    ref, _ = oracle_mod.decode_rows(u16(host["q"]), u16(host["k_cache"]), u16(host["v_cache"]),
                                    host["block_table"].numpy(), host["seq_lens"].numpy(),
                                    host["bias"].numpy(), window, spec.D_max)
    for call in range(2):
        out = torch.full_like(t["q"], float("nan"))
        _static_c(t, window, out, 0)
        torch.cuda.synchronize()
        assert_parity(out, ref, f"static decode, window {window}, call {call}")


def test_static_scratch_runs_the_whole_and_pieces_plan(oracle_mod):
    """48 sequences x 3 draft tokens fill the SMs' slots: the automatic plan
    runs the first sequences unsplit and the rest in pieces, and its partials
    (a few MB) fit the library's array.  Two calls in a row equal
    inkling_attn_decode with a workspace bit for bit, and the oracle on every
    row."""
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=48, L_min=200, L_max=3000, window=1000,
                  n_new=3, seed=24)
    t = make_decode(spec, device="cuda")
    assert ink.decode_num_splits(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                 t["seq_lens"], t["bias"], window=spec.window) > 1
    ref_ws = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                             t["seq_lens"], t["bias"], window=spec.window)
    host = {k: v.cpu() for k, v in t.items()}
    ref, _ = oracle_mod.decode_mq_rows(u16(host["q"]), u16(host["k_cache"]),
                                       u16(host["v_cache"]), host["block_table"].numpy(),
                                       host["seq_lens"].numpy(), host["bias"].numpy(),
                                       spec.window, spec.D_max)
    for call in range(2):
        out = torch.full_like(t["q"], float("nan"))
        _static_c(t, spec.window, out, 0)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_ws), f"call {call}: differs from the workspace call"
        assert_parity(out, ref, f"whole + pieces static decode, call {call}")


def test_static_scratch_lowers_the_automatic_split_count(oracle_mod):
    """Multi-token decode (10 draft tokens) of 2 sequences of 40,000 tokens:
    the automatic split count needs more partials than the 8 MiB array holds,
    so the call lowers it to the largest count that fits.  Checked against
    inkling_attn_decode with a workspace at that count (same kernels, same
    result bit for bit) and against the oracle on every row."""
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=2, L_min=40000, L_max=40000, window=0,
                  D_max=65536, n_new=10, seed=22)
    t = make_decode(spec, device="cuda")
    S, Q, Hq = spec.S, spec.n_new, spec.Hq
    auto = ink.decode_num_splits(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                                 t["seq_lens"], t["bias"], window=0)
    cap = 8 << 20
    assert ink.decode_workspace_bytes(S * Q, Hq, auto) > cap, "case must exceed the array"
    lowered = auto
    while lowered > 1 and ink.decode_workspace_bytes(S * Q, Hq, lowered) > cap:
        lowered -= 1
    assert 1 < lowered < auto
    ref_ws = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"],
                             t["seq_lens"], t["bias"], window=0, num_splits=lowered)
    host = {k: v.cpu() for k, v in t.items()}
    ref, _ = oracle_mod.decode_mq_rows(u16(host["q"]), u16(host["k_cache"]),
                                       u16(host["v_cache"]), host["block_table"].numpy(),
                                       host["seq_lens"].numpy(), host["bias"].numpy(), 0,
                                       spec.D_max)
    for call in range(2):
        out = torch.full_like(t["q"], float("nan"))
        _static_c(t, 0, out, 0)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_ws), f"call {call}: differs from the workspace call"
        assert_parity(out, ref, f"lowered static decode, call {call}")


@pytest.mark.parametrize("q_len,splits", [(1, 4), (3, 4), (1, 16), (3, 16)])
def test_static_scratch_rows_that_cannot_be_computed_read_nan(q_len, splits):
    """A call whose sequence 1 has a length outside [q_len, max_blocks*128]
    reports BAD_LENGTH and writes NaN for that sequence's rows (never the
    previous call's partials, which are still in the array); the other
    sequences' rows equal those of a valid call.  4 splits merge with one
    warp per row, 16 with four."""
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=4, L_min=5000, L_max=9000, window=0,
                  n_new=q_len, seed=23)
    t = make_decode(spec, device="cuda")
    first = torch.empty_like(t["q"])
    _static_c(t, 0, first, splits)   # fills the array with this call's partials
    bad = dict(t)
    bad["seq_lens"] = t["seq_lens"].clone()
    bad["seq_lens"][1] = t["block_table"].shape[1] * 128 + 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(t["q"])
    _static_c(bad, 0, out, splits, status=status)
    torch.cuda.synchronize()
    assert status.item() & binding.STATUS_BAD_LENGTH
    assert torch.isnan(out[1].float()).all()
    keep = [0, 2, 3]
    assert torch.equal(out[keep], first[keep])
