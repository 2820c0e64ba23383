"""The benchmark's algorithmic work (allowed pairs, FLOPs, key/value bytes) and
the input recipe, checked against brute-force counts and closed forms."""
import numpy as np
import pytest
import torch

from relative_bias_sliding_b200.inputs import (WORKLOADS, ChunkSpec, DecodeSpec, PrefillSpec,
                                               kv_bytes_read, make_chunk, make_prefill, scaled)


def _pairs_brute(T, W, rows=None):
    """(i, j) with 0 <= i - j (< W when W > 0), i over `rows` (default all)."""
    i = np.arange(T)[:, None] if rows is None else np.asarray(rows)[:, None]
    j = np.arange(T)[None, :]
    d = i - j
    ok = d >= 0
    if W > 0:
        ok &= d < W
    return int(ok.sum())


@pytest.mark.parametrize("T,W", [(1, 0), (7, 0), (300, 0), (300, 1), (300, 128), (300, 299),
                                 (300, 300), (300, 1000), (1000, 257)])
def test_prefill_pairs_match_brute_force(T, W):
    spec = PrefillSpec("t", 1, T, 8, 1, 128, W, 64, 1.0, 0)
    assert spec.allowed_pairs == _pairs_brute(T, W)
    assert spec.flops == 4 * 128 * 8 * spec.allowed_pairs


def test_headline_work():
    swa, full = WORKLOADS["prefill_swa_b4_t8192"], WORKLOADS["prefill_full_b1_t32768"]
    # window 4096 over 8192 tokens: W(W+1)/2 + (T-W)W pairs per (b, h)
    assert swa.allowed_pairs == 4096 * 4097 // 2 + 4096 * 4096 == 25_167_872
    assert swa.flops == 4 * 128 * 64 * 4 * 25_167_872 == 3_298_803_318_784
    assert full.allowed_pairs == 32768 * 32769 // 2 == 536_887_296
    assert full.flops == 4 * 128 * 64 * 536_887_296


@pytest.mark.parametrize("prefix,chunk,W", [(0, 300, 0), (0, 300, 100), (500, 37, 0),
                                            (500, 37, 128), (6144, 64, 4096), (1, 1, 1)])
def test_chunk_pairs_are_the_chunk_rows_of_the_prefill(prefix, chunk, W):
    spec = ChunkSpec("c", 1, prefix, chunk, 8, 1, 128, W, 64, 1.0, 0)
    T = prefix + chunk
    assert spec.allowed_pairs == _pairs_brute(T, W, rows=range(prefix, T))
    if prefix == 0:
        assert spec.allowed_pairs == PrefillSpec("p", 1, T, 8, 1, 128, W, 64, 1.0, 0).allowed_pairs


def test_paged_workload_has_the_dense_workload_flops():
    assert (WORKLOADS["prefill_paged_swa_b4_t8192"].flops ==
            WORKLOADS["prefill_swa_b4_t8192"].flops)


@pytest.mark.parametrize("W,n_new", [(0, 1), (100, 1), (100, 9), (4096, 1), (4096, 9)])
def test_decode_kv_bytes_are_the_union_of_the_windows(W, n_new):
    spec = DecodeSpec("d", 4, 50, 5000, 64, 8, 128, W, 4096, 1.0, 0, n_new=n_new)
    lens = torch.tensor([50, 99, 100, 5000], dtype=torch.int32)
    keys = 0
    for L in lens.tolist():
        seen = set()
        for qi in range(n_new):
            i = L - n_new + qi
            lo = max(0, i - W + 1) if W > 0 else 0
            seen.update(range(lo, i + 1))
        keys += len(seen)
    assert kv_bytes_read(spec, lens) == keys * 8 * 128 * 2 * 2


def test_inputs_are_seeded_and_follow_the_recipe():
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], T=64)
    a, b = make_prefill(spec), make_prefill(spec)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (1, 64, 8, 128)
    assert a["w_k"].shape == (128, 4) and a["bias"].shape == (8, spec.D_max + 1)
    # N(0, 1) activations, N(0, 0.5) taps (0.5 is the standard deviation)
    assert abs(a["q"].float().std().item() - 1.0) < 0.05
    assert abs(a["w_k"].std().item() - 0.5) < 0.1
    other = make_prefill(scaled(spec, seed=spec.seed + 1))
    assert not torch.equal(a["q"], other["q"])


def test_chunk_inputs_of_an_empty_sequence_have_zero_history():
    spec = scaled(WORKLOADS["prefill_paged_swa_b4_t8192"], B=2, chunk=200)
    t = make_chunk(spec)
    assert not t["k_state"].any() and not t["v_state"].any()
    assert t["seq_lens"].tolist() == [200, 200]
    assert t["cu_q"].tolist() == [0, 200, 400]
    # every sequence's blocks are distinct entries of the pool
    bt = t["block_table"].flatten().tolist()
    assert len(set(bt)) == len(bt) and max(bt) < t["k_cache"].shape[0]
    with_prefix = make_chunk(scaled(WORKLOADS["prefill_chunked_swa_b4_c2048"], B=2, prefix=300,
                                    chunk=50))
    assert with_prefix["k_state"].any()
