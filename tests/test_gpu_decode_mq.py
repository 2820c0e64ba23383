"""Multi-token paged decode (draft tokens of speculative decoding / multi-token
prediction) on the GPU against the oracle, plus invariants."""
import numpy as np
import pytest
import torch

from conftest import assert_parity, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import (WORKLOADS, BLOCK, make_decode, make_prefill,
                                               scaled)

pytestmark = pytest.mark.gpu


def _inputs(S, Q, lens, Hq=64, Hkv=8, d_max=4096, seed=0, extra=5):
    g = torch.Generator().manual_seed(seed)
    d = 128
    q = torch.randn((S, Q, Hq, d), generator=g).to(torch.bfloat16)
    bias = torch.randn((Hq, d_max + 1), generator=g)
    nb = [(L + BLOCK - 1) // BLOCK for L in lens]
    total = sum(nb) + extra
    perm = torch.randperm(total, generator=g).to(torch.int32)
    bt = torch.zeros((S, max(nb)), dtype=torch.int32)
    off = 0
    for s in range(S):
        bt[s, :nb[s]] = perm[off:off + nb[s]]
        off += nb[s]
    kc = torch.randn((total, Hkv, BLOCK, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((total, Hkv, BLOCK, d), generator=g).to(torch.bfloat16)
    return dict(q=q, k_cache=kc, v_cache=vc, block_table=bt,
                seq_lens=torch.tensor(lens, dtype=torch.int32), bias=bias)


def _oracle(oracle_mod, t, window, rows=None):
    return oracle_mod.decode_mq_rows(u16(t["q"]), u16(t["k_cache"]), u16(t["v_cache"]),
                                     t["block_table"].numpy(), t["seq_lens"].numpy(),
                                     t["bias"].numpy(), window, t["bias"].shape[1] - 1, rows)


def _gpu(t, window, num_splits=0):
    dev = {k: v.cuda() for k, v in t.items()}
    lse = torch.empty(dev["q"].shape[:-1], dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ink.attn_decode(**dev, window=window, lse=lse, num_splits=num_splits, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0, f"status {status.item()}"
    return out, lse


@pytest.mark.parametrize("Q", [2, 3, 5, 9])
@pytest.mark.parametrize("window,splits", [(0, 1), (0, 3), (100, 0), (1000, 2), (0, 9), (0, 33)])
def test_decode_mq_matches_oracle(oracle_mod, Q, window, splits):
    need_gpu()
    # lengths from exactly Q (every key is a draft token) to several blocks,
    # including chunk and block boundaries
    lens = [Q, Q + 1, 64, 65, 129, 700, 2100]
    t = _inputs(len(lens), Q, lens, Hq=16, Hkv=2, d_max=300, seed=10 * Q + splits + window)
    ref, ref_lse = _oracle(oracle_mod, t, window)
    out, lse = _gpu(t, window, splits)
    assert_parity(out, ref, f"Q={Q} W={window} splits={splits}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, rtol=0, atol=2e-3)


@pytest.mark.parametrize("G,Q", [(1, 10), (2, 9), (4, 7), (8, 9), (8, 10), (5, 4)])
def test_decode_mq_group_sizes(oracle_mod, G, Q):
    """(query heads per kv head) x q_len rows are cut into 16-row tiles: full,
    partial and a group size that does not divide 16."""
    need_gpu()
    lens = [300, 1500, Q + 5]
    t = _inputs(3, Q, lens, Hq=2 * G, Hkv=2, d_max=64, seed=G * 100 + Q)
    ref, _ = _oracle(oracle_mod, t, 0)
    out, _ = _gpu(t, 0, 2)
    assert_parity(out, ref, f"G={G} Q={Q}")


def test_decode_mq_first_token_equals_single_token_decode():
    """Query 0 of q_len draft tokens at length L sees exactly what a
    single-token decode at length L - q_len + 1 sees."""
    need_gpu()
    Q = 9
    lens = [900, 4096 + 9, 77]
    t = _inputs(3, Q, lens, Hq=16, Hkv=2, d_max=4096, seed=4)
    mq, _ = _gpu(t, 1000, 3)
    one = dict(t)
    one["q"] = t["q"][:, 0].contiguous()
    one["seq_lens"] = t["seq_lens"] - (Q - 1)
    dev = {k: v.cuda() for k, v in one.items()}
    single = ink.attn_decode(**dev, window=1000, num_splits=3)
    torch.cuda.synchronize()
    assert (mq[:, 0].float() - single.float()).abs().max().item() < 2e-2


def test_decode_mq_rows_equal_prefill_rows(oracle_mod):
    """The last q_len prefill rows equal a multi-token decode over the cache
    that sconv_kv builds from the same raw keys and values."""
    need_gpu()
    T, Hq, Hkv, W, D, Q = 1000, 16, 2, 300, 512, 9
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], T=T, Hq=Hq, Hkv=Hkv, window=W, D_max=D,
                  seed=3)
    t = make_prefill(spec)
    dev = {k: v.cuda() for k, v in t.items()}
    pre = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                           dev["bias"], window=W)
    nb = (T + 127) // 128
    kc = torch.zeros((nb + 2, Hkv, 128, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    bt = torch.arange(2, nb + 2, dtype=torch.int32, device="cuda")[None]
    ks = torch.zeros((1, 3, Hkv * 128), dtype=torch.bfloat16, device="cuda")
    vs = torch.zeros_like(ks)
    done = 0
    while done < T:   # the last append is the Q draft tokens
        n = min(64, T - Q - done) if done < T - Q else Q
        ink.sconv_kv(dev["k_raw"][:, done:done + n].contiguous(),
                     dev["v_raw"][:, done:done + n].contiguous(), dev["w_k"], dev["w_v"], ks, vs,
                     kc, vc, bt, torch.tensor([done + n], dtype=torch.int32, device="cuda"))
        done += n
    dec = ink.attn_decode(dev["q"][:, T - Q:].contiguous(), kc, vc, bt,
                          torch.tensor([T], dtype=torch.int32, device="cuda"), dev["bias"],
                          window=W, num_splits=2)
    torch.cuda.synchronize()
    assert (dec.float() - pre[:, T - Q:].float()).abs().max().item() < 2e-2
    rows = np.array([[0, h, i] for i in range(T - Q, T) for h in range(Hq)], np.int32)
    ref, _, _, _ = oracle_mod.prefill_rows(u16(t["q"]), u16(t["k_raw"]), u16(t["v_raw"]),
                                           t["w_k"].numpy(), t["w_v"].numpy(), t["bias"].numpy(),
                                           W, D, rows)
    assert_parity(dec[0], ref, "multi-token decode vs oracle prefill rows")


def test_decode_mq_static_matches_workspace_call():
    need_gpu()
    Q = 9
    lens = [5000, 300, 4096]
    t = _inputs(3, Q, lens, Hq=64, Hkv=8, d_max=4096, seed=8)
    dev = {k: v.cuda() for k, v in t.items()}
    a = ink.attn_decode(**dev, window=4096)
    b = ink.attn_decode_static(**dev, window=4096)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_decode_mq_whole_and_split_sequences_match_oracle(oracle_mod):
    """48 sequences x 8 kv heads fill the SMs' slots: the automatic plan runs
    the sequences that fill whole waves unsplit and the rest in key-range
    pieces merged by the combine (reported split count > 1).  Every row and
    lse against the oracle."""
    need_gpu()
    S, Q = 48, 3
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(Q, 1500, size=S)]
    t = _inputs(S, Q, lens, Hq=64, Hkv=8, d_max=1024, seed=55)
    dev = {k: v.cuda() for k, v in t.items()}
    reported = ink.decode_num_splits(dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                                     dev["seq_lens"], dev["bias"], window=0)
    assert reported > 1, "the case must take the whole + pieces plan"
    ref, ref_lse = _oracle(oracle_mod, t, 0)
    out, lse = _gpu(t, 0)
    assert_parity(out, ref, "whole + pieces plan")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, rtol=0, atol=2e-3)
    # the same call with one split (no partials) agrees with it closely
    one, _ = _gpu(t, 0, 1)
    assert (one.float() - out.float()).abs().max().item() < 1e-2


def test_decode_mq_whole_and_split_bad_length_rows_read_nan():
    """With the whole + pieces plan, a sequence of bad length among the whole
    ones and one among the split ones both read NaN; the others are those of
    a valid call."""
    need_gpu()
    S, Q = 48, 2
    rng = np.random.default_rng(6)
    lens = [int(x) for x in rng.integers(Q, 900, size=S)]
    t = _inputs(S, Q, lens, Hq=64, Hkv=8, d_max=1024, seed=56)
    good, _ = _gpu(t, 0)
    bad = dict(t)
    bad["seq_lens"] = t["seq_lens"].clone()
    bad["seq_lens"][0] = 1           # a whole sequence: fewer than q_len tokens
    bad["seq_lens"][S - 1] = 1       # a split sequence
    dev = {k: v.cuda() for k, v in bad.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ink.attn_decode(**dev, window=0, status=status)
    torch.cuda.synchronize()
    assert status.item() & 4   # INKLING_STATUS_BAD_LENGTH
    assert torch.isnan(out[0].float()).all() and torch.isnan(out[S - 1].float()).all()
    assert torch.equal(out[1:S - 1], good[1:S - 1])


def test_decode_mq_rejects_too_many_rows():
    need_gpu()
    t = _inputs(1, 11, [100], Hq=16, Hkv=2, d_max=64)   # G 8 x 11 tokens = 88 rows
    dev = {k: v.cuda() for k, v in t.items()}
    with pytest.raises(ink.InklingError):
        ink.attn_decode(**dev, window=0)


def test_decode_mq_short_sequence_reports_bad_length():
    need_gpu()
    t = _inputs(2, 9, [100, 100], Hq=16, Hkv=2, d_max=64)
    t["seq_lens"] = torch.tensor([100, 5], dtype=torch.int32)   # fewer than q_len tokens
    dev = {k: v.cuda() for k, v in t.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ink.attn_decode(**dev, window=0, status=status, num_splits=1)
    torch.cuda.synchronize()
    assert status.item() & 4   # INKLING_STATUS_BAD_LENGTH


@pytest.mark.parametrize("per_seq", [4])
def test_decode_mtp9_workload_sampled_rows(oracle_mod, per_seq):
    """The sliding-window decode workload verifying 9 draft tokens: sconv
    append of the 9 tokens, then multi-token decode; sampled (seq, token, head)
    rows against the oracle."""
    need_gpu()
    spec = WORKLOADS["decode_mtp9_swa_s64"]
    t = make_decode(spec)
    dev = {k: v.cuda() for k, v in t.items()}
    ink.sconv_kv(dev["k_new"], dev["v_new"], dev["w_k"], dev["w_v"], dev["k_state"],
                 dev["v_state"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                 dev["seq_lens"])
    out = ink.attn_decode(dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                          dev["seq_lens"], dev["bias"], window=spec.window)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    rows = np.array([[s, rng.integers(0, spec.n_new), rng.integers(0, spec.Hq)]
                     for s in range(spec.S) for _ in range(per_seq)], np.int32)
    host = {k: v.cpu() for k, v in dev.items()}
    ref, _ = oracle_mod.decode_mq_rows(u16(host["q"]), u16(host["k_cache"]), u16(host["v_cache"]),
                                       host["block_table"].numpy(), host["seq_lens"].numpy(),
                                       host["bias"].numpy(), spec.window, spec.D_max, rows)
    got = out.cpu()[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_parity(got, ref, "decode_mtp9_swa_s64 sampled rows")
