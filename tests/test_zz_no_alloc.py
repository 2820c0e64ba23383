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

from conftest import MAX_ABS, REL_L2, errors, need_gpu
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
