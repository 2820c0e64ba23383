"""Failure detection without a GPU fault: a bounded wait inside a kernel runs
out, the kernel reports INKLING_STATUS_TIMEOUT through the status word and
returns, and the CUDA context keeps working."""
import time

import pytest
import torch

from conftest import need_gpu
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200 import binding
from relative_bias_sliding_b200.inputs import WORKLOADS, make_decode, scaled

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    need_gpu()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    binding.selftest_wait_timeout(status, limit_us=50000)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert status.item() & binding.STATUS_TIMEOUT
    assert elapsed < 5.0
    # the context is still usable: a normal decode runs and is self-consistent
    spec = scaled(WORKLOADS["decode_swa_s64"], S=3, L_min=200, L_max=900, window=0, D_max=1000)
    t = make_decode(spec, device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    a = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                        t["bias"], num_splits=1, status=st2)
    b = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                        t["bias"], num_splits=1)
    torch.cuda.synchronize()
    assert st2.item() == 0
    assert torch.equal(a, b) and torch.isfinite(a.float()).all()


def test_selftest_rejects_bad_arguments():
    need_gpu()
    lib = binding.load_library()
    assert lib.inkling_selftest_wait_timeout(None, 100, None) == binding.INKLING_ERR_INVALID
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.inkling_selftest_wait_timeout(binding._ptr(status), 0, None) == \
        binding.INKLING_ERR_INVALID
