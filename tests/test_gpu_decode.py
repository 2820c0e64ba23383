"""Split-KV paged decode on the GPU against the oracle, plus invariants."""
import numpy as np
import pytest
import torch

from conftest import assert_parity, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import WORKLOADS, BLOCK, make_decode, scaled

pytestmark = pytest.mark.gpu


def _inputs(S, lens, Hq=64, Hkv=8, window=0, d_max=4096, seed=0, extra=5, bias_std=1.0):
    g = torch.Generator().manual_seed(seed)
    d = 128
    q = torch.randn((S, Hq, d), generator=g).to(torch.bfloat16)
    bias = torch.randn((Hq, d_max + 1), generator=g) * bias_std
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
                seq_lens=torch.tensor(lens, dtype=torch.int32), bias=bias), window


def _oracle(oracle_mod, t, window, pairs=None):
    S, Hq, d = t["q"].shape
    out, lse = oracle_mod.decode_rows(u16(t["q"]), u16(t["k_cache"]), u16(t["v_cache"]),
                                      t["block_table"].numpy(), t["seq_lens"].numpy(),
                                      t["bias"].numpy(), window, t["bias"].shape[1] - 1, pairs)
    return out, lse


def _gpu(t, window, num_splits=0, with_lse=True):
    dev = {k: v.cuda() for k, v in t.items()}
    S, Hq, _ = dev["q"].shape
    lse = torch.empty((S, Hq), dtype=torch.float32, device="cuda") if with_lse else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ink.attn_decode(**dev, window=window, lse=lse, num_splits=num_splits, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out, lse


@pytest.mark.parametrize("window", [0, 100, 4096])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_decode_small_matches_oracle(oracle_mod, window, splits):
    need_gpu()
    lens = [1, 2, 63, 64, 65, 128, 129, 1000, 4097, 5000]
    t, W = _inputs(len(lens), lens, Hq=16, Hkv=2, window=window, d_max=300, seed=splits + window)
    ref, ref_lse = _oracle(oracle_mod, t, W)
    out, lse = _gpu(t, W, splits)
    assert_parity(out, ref, f"W={window} splits={splits}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, rtol=0, atol=2e-3)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_gqa_group_sizes(oracle_mod, G):
    need_gpu()
    lens = [300, 77, 1500]
    t, W = _inputs(3, lens, Hq=2 * G, Hkv=2, window=0, d_max=64, seed=G)
    ref, _ = _oracle(oracle_mod, t, W)
    out, _ = _gpu(t, W, 2)
    assert_parity(out, ref, f"G={G}")


def test_decode_block_permutation_is_bit_exact():
    need_gpu()
    lens = [700, 3000, 129]
    t, W = _inputs(3, lens, Hq=16, Hkv=2, window=0, d_max=4096, seed=7, extra=20)
    out1, _ = _gpu(t, W, 4)
    # move every block to a new physical slot, copy contents, rewrite the table
    total = t["k_cache"].shape[0]
    perm = torch.randperm(total, generator=torch.Generator().manual_seed(3))
    t2 = dict(t)
    t2["k_cache"] = torch.empty_like(t["k_cache"])
    t2["v_cache"] = torch.empty_like(t["v_cache"])
    t2["k_cache"][perm] = t["k_cache"]
    t2["v_cache"][perm] = t["v_cache"]
    t2["block_table"] = perm[t["block_table"].long()].to(torch.int32)
    out2, _ = _gpu(t2, W, 4)
    assert torch.equal(out1, out2)


def test_decode_whole_and_split_sequences_match_oracle(oracle_mod):
    """48 sequences x 8 kv heads fill the SMs' slots: the automatic plan runs
    the sequences that fill whole waves unsplit and the rest in key-range
    pieces merged by the combine (reported split count > 1).  Every (seq,
    head) row and lse against the oracle; a sequence of bad length among the
    whole ones and one among the split ones read NaN."""
    need_gpu()
    S = 48
    rng = np.random.default_rng(8)
    lens = [int(x) for x in rng.integers(1, 3000, size=S)]
    t, W = _inputs(S, lens, Hq=64, Hkv=8, window=0, d_max=2048, seed=58)
    dev = {k: v.cuda() for k, v in t.items()}
    reported = ink.decode_num_splits(dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                                     dev["seq_lens"], dev["bias"], window=0)
    assert reported > 1, "the case must take the whole + pieces plan"
    ref, ref_lse = _oracle(oracle_mod, t, W)
    out, lse = _gpu(t, W)
    assert_parity(out, ref, "whole + pieces plan")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, rtol=0, atol=2e-3)
    bad = dict(t)
    bad["seq_lens"] = t["seq_lens"].clone()
    bad["seq_lens"][0] = 0
    bad["seq_lens"][S - 1] = 0
    bdev = {k: v.cuda() for k, v in bad.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out2 = ink.attn_decode(**bdev, window=0, status=status)
    torch.cuda.synchronize()
    assert status.item() & 4   # INKLING_STATUS_BAD_LENGTH
    assert torch.isnan(out2[0].float()).all() and torch.isnan(out2[S - 1].float()).all()
    assert torch.equal(out2[1:S - 1], out[1:S - 1])


@pytest.mark.parametrize("splits", [8, 12, 20, 40])
def test_decode_combine_warps_per_row_matches_oracle(oracle_mod, splits):
    """The combine merges each row with 1, 2, 4 or 8 warps by split count:
    each width against the oracle, with empty splits (a 130-token sequence)
    in the mix."""
    need_gpu()
    lens = [9000, 130, 20000]
    t, W = _inputs(3, lens, Hq=16, Hkv=2, window=0, d_max=30000, seed=40 + splits)
    ref, ref_lse = _oracle(oracle_mod, t, W)
    out, lse = _gpu(t, W, splits)
    assert_parity(out, ref, f"splits={splits}")
    np.testing.assert_allclose(lse.cpu().numpy().reshape(-1), ref_lse, rtol=0, atol=2e-3)


def test_decode_split_count_invariance():
    need_gpu()
    lens = [9000, 130, 4500]
    t, W = _inputs(3, lens, Hq=16, Hkv=2, window=0, d_max=10000, seed=9)
    outs = [_gpu(t, W, s)[0].float() for s in (1, 2, 5, 17)]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() < 1e-2


def test_decode_swa_workload_full_size(oracle_mod):
    """The sliding-window decode workload (64 sequences, lengths U[1024, 32768],
    window 4096) at full size in the benchmark's launch configuration: the
    sconv append of the new token, then split-KV decode; every (sequence,
    head) pair checked against the oracle."""
    need_gpu()
    spec = WORKLOADS["decode_swa_s64"]
    t = make_decode(spec, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    host = {k: v.cpu() for k, v in t.items()}
    ink.sconv_kv(t["k_new"], t["v_new"], t["w_k"], t["w_v"], t["k_state"], t["v_state"],
                 t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"], status=status)
    out = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                          t["bias"], window=spec.window, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # oracle: append on host copies, then decode
    kc, vc = u16(host["k_cache"]).copy(), u16(host["v_cache"]).copy()
    ks, vs = u16(host["k_state"]).copy(), u16(host["v_state"]).copy()
    oracle_mod.sconv_append(u16(host["k_new"]), ks, host["w_k"].numpy(), kc,
                            host["block_table"].numpy(), host["seq_lens"].numpy())
    oracle_mod.sconv_append(u16(host["v_new"]), vs, host["w_v"].numpy(), vc,
                            host["block_table"].numpy(), host["seq_lens"].numpy())
    ref, _ = oracle_mod.decode_rows(u16(host["q"]), kc, vc, host["block_table"].numpy(),
                                    host["seq_lens"].numpy(), host["bias"].numpy(), spec.window,
                                    spec.D_max)
    assert_parity(out, ref, "decode_swa_s64")


@pytest.mark.parametrize("name", ["decode_full_1m_b1", "decode_full_1m_b8"])
def test_decode_long_context_sampled(oracle_mod, name):
    """1M-token full-attention decode at full size; the oracle checks every
    query head of the first and last sequence, through a host copy of those
    sequences' blocks."""
    need_gpu()
    spec = WORKLOADS[name]
    t = make_decode(spec, device="cuda")
    out = ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                          t["bias"], window=0)
    torch.cuda.synchronize()
    seqs = [0] if spec.S == 1 else [0, spec.S - 1]
    heads = list(range(spec.Hq))
    for s in seqs:
        ids = t["block_table"][s].long()
        kc = u16(t["k_cache"][ids])                    # this sequence's blocks, in order
        vc = u16(t["v_cache"][ids])
        bt = np.arange(len(ids), dtype=np.int32)[None, :]
        L = np.array([int(t["seq_lens"][s])], np.int32)
        pairs = np.array([[0, h] for h in heads], np.int32)
        ref, _ = oracle_mod.decode_rows(u16(t["q"][s:s + 1]), kc, vc, bt, L,
                                        t["bias"].cpu().numpy(), 0, spec.D_max, pairs)
        got = out[s, heads].float().cpu().numpy()
        assert_parity(got, ref, f"{name} seq {s}")
        del kc, vc
