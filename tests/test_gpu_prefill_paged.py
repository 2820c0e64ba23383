"""Chunked prefill over the paged cache (sconv_kv append of each chunk, then
attn_prefill_paged) on the GPU: the rows of every chunk equal the prefill of
the whole sequence (oracle, and the dense GPU prefill)."""
import numpy as np
import pytest
import torch

from conftest import assert_append_close, assert_parity, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import BLOCK, WORKLOADS as WORKLOADS_CHUNK

pytestmark = pytest.mark.gpu


def _sequences(lens, Hq, Hkv, D_max, seed):
    g = torch.Generator().manual_seed(seed)
    d, C = 128, Hkv * 128
    seqs = []
    for T in lens:
        seqs.append(dict(q=torch.randn((1, T, Hq, d), generator=g).to(torch.bfloat16),
                         k=torch.randn((1, T, Hkv, d), generator=g).to(torch.bfloat16),
                         v=torch.randn((1, T, Hkv, d), generator=g).to(torch.bfloat16)))
    w_k = torch.randn((C, 4), generator=g) * 0.5
    w_v = torch.randn((C, 4), generator=g) * 0.5
    bias = torch.randn((Hq, D_max + 1), generator=g)
    return seqs, w_k, w_v, bias


def _chunked(seqs, w_k, w_v, bias, chunks, window, Hkv, extra_blocks=3, seed=0):
    """Run the chunk schedule: chunks[c][s] new tokens of sequence s in step c.
    Returns per-sequence outputs [T, Hq, d] (bf16, CUDA) and lse [T, Hq]."""
    S = len(seqs)
    Hq = seqs[0]["q"].shape[2]
    lens = [x["q"].shape[1] for x in seqs]
    nb = [(T + BLOCK - 1) // BLOCK for T in lens]
    total = sum(nb) + extra_blocks
    perm = torch.randperm(total, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    bt = torch.zeros((S, max(nb)), dtype=torch.int32)
    off = 0
    for s in range(S):
        bt[s, :nb[s]] = perm[off:off + nb[s]]
        off += nb[s]
    bt = bt.cuda()
    kc = torch.randn((total, Hkv, BLOCK, 128), device="cuda").to(torch.bfloat16)  # stale contents
    vc = torch.randn((total, Hkv, BLOCK, 128), device="cuda").to(torch.bfloat16)
    ks = torch.zeros((S, 3, Hkv * 128), dtype=torch.bfloat16, device="cuda")
    vs = torch.zeros_like(ks)
    wk, wv, b = w_k.cuda(), w_v.cuda(), bias.cuda()
    outs = [torch.empty((T, Hq, 128), dtype=torch.bfloat16, device="cuda") for T in lens]
    lses = [torch.empty((T, Hq), dtype=torch.float32, device="cuda") for T in lens]
    done = [0] * S
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in chunks:
        n = [min(step[s], lens[s] - done[s]) for s in range(S)]
        # append each sequence's chunk (sconv continues from its state)
        for s in range(S):
            if n[s] == 0:
                continue
            sl = slice(done[s], done[s] + n[s])
            ink.sconv_kv(seqs[s]["k"][:, sl].contiguous().cuda(),
                         seqs[s]["v"][:, sl].contiguous().cuda(), wk, wv, ks[s:s + 1],
                         vs[s:s + 1], kc, vc, bt[s:s + 1],
                         torch.tensor([done[s] + n[s]], dtype=torch.int32, device="cuda"),
                         status=status)
        cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
        if cu[-1] == 0:
            continue
        q = torch.cat([seqs[s]["q"][0, done[s]:done[s] + n[s]] for s in range(S)]).cuda()
        lse = torch.empty((q.shape[0], Hq), dtype=torch.float32, device="cuda")
        seq_lens = torch.tensor([done[s] + n[s] for s in range(S)], dtype=torch.int32,
                                device="cuda")
        out = ink.attn_prefill_paged(q, torch.from_numpy(cu).cuda(), kc, vc, bt, seq_lens, b,
                                     window=window, lse=lse, status=status)
        for s in range(S):
            outs[s][done[s]:done[s] + n[s]] = out[cu[s]:cu[s + 1]]
            lses[s][done[s]:done[s] + n[s]] = lse[cu[s]:cu[s + 1]]
            done[s] += n[s]
    torch.cuda.synchronize()
    assert status.item() == 0, f"status {status.item()}"
    assert done == lens
    return outs, lses


@pytest.mark.parametrize("Hq,Hkv,window,D_max", [
    (8, 1, 0, 2000),     # G = 8, full causal
    (6, 2, 300, 256),    # G = 3, window, clip inside the band
    (4, 4, 128, 1000),   # G = 1, window of exactly one tile
    (4, 2, 500, 600),    # G = 2: two heads x 128 rows per block, window, clip
    (12, 2, 0, 1500),    # G = 6: three head pairs per kv head, full causal
])
def test_chunked_prefill_equals_whole_sequence_oracle(oracle_mod, Hq, Hkv, window, D_max):
    need_gpu()
    lens = [700, 1, 300, 1029]
    seqs, w_k, w_v, bias = _sequences(lens, Hq, Hkv, D_max, seed=Hq + window)
    # uneven chunks per sequence and step, including empty ones, a single
    # token, chunks that straddle block and query-block boundaries
    chunks = [[256, 1, 0, 129], [1, 0, 300, 256], [300, 0, 0, 1], [143, 0, 0, 643]]
    outs, lses = _chunked(seqs, w_k, w_v, bias, chunks, window, Hkv, seed=1)
    for s, x in enumerate(seqs):
        ref, ref_lse, _, _ = oracle_mod.prefill_rows(u16(x["q"]), u16(x["k"]), u16(x["v"]),
                                                     w_k.numpy(), w_v.numpy(), bias.numpy(),
                                                     window, D_max)
        assert_parity(outs[s], ref, f"seq {s} (T={lens[s]})")
        np.testing.assert_allclose(lses[s].cpu().numpy().reshape(-1), ref_lse, rtol=0, atol=2e-3)


def test_chunked_prefill_matches_dense_prefill():
    """One sequence in chunks of 1000 vs the dense fused-sconv prefill."""
    need_gpu()
    T, Hq, Hkv, W, D = 4000, 16, 2, 1500, 4096
    seqs, w_k, w_v, bias = _sequences([T], Hq, Hkv, D, seed=7)
    outs, _ = _chunked(seqs, w_k, w_v, bias, [[1000]] * 4, W, Hkv, seed=2)
    x = seqs[0]
    dense = ink.attn_prefill(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), w_k.cuda(), w_v.cuda(),
                             bias.cuda(), window=W)
    torch.cuda.synchronize()
    assert (outs[0].float() - dense[0].float()).abs().max().item() < 2e-2


def test_chunked_prefill_reports_short_length():
    need_gpu()
    Hq, Hkv = 8, 1
    q = torch.randn((10, Hq, 128), device="cuda").to(torch.bfloat16)
    kc = torch.zeros((2, Hkv, BLOCK, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ink.attn_prefill_paged(q, torch.tensor([0, 10], dtype=torch.int32, device="cuda"), kc, kc,
                           bt, torch.tensor([5], dtype=torch.int32, device="cuda"),
                           torch.zeros((Hq, 17), device="cuda"), status=status)
    torch.cuda.synchronize()
    assert status.item() & 4   # INKLING_STATUS_BAD_LENGTH: 10 new tokens, length 5


@pytest.mark.parametrize("name", ["prefill_chunked_swa_b4_c2048", "prefill_paged_swa_b4_t8192"])
def test_chunked_workload_sampled_rows(oracle_mod, name):
    """The chunked-prefill bench workloads (4 sequences with a 6144-token
    prefix and a 2048-token chunk; 4 empty sequences taking 8192 tokens;
    window 4096): GPU append + paged prefill; sampled (row, head) pairs against
    the oracle's append + paged attention of the same rows (query r at
    position prefix + r)."""
    need_gpu()
    from relative_bias_sliding_b200.inputs import make_chunk
    spec = WORKLOADS_CHUNK[name]
    t = make_chunk(spec)
    host = {k: v.clone() for k, v in t.items()}
    dev = {k: v.cuda() for k, v in t.items()}
    ink.sconv_kv(dev["k_new"], dev["v_new"], dev["w_k"], dev["w_v"], dev["k_state"],
                 dev["v_state"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                 dev["seq_lens"])
    out = ink.attn_prefill_paged(dev["q"], dev["cu_q"], dev["k_cache"], dev["v_cache"],
                                 dev["block_table"], dev["seq_lens"], dev["bias"],
                                 window=spec.window, max_q=spec.chunk)
    torch.cuda.synchronize()
    kc, vc = u16(host["k_cache"]).copy(), u16(host["v_cache"]).copy()
    ks, vs = u16(host["k_state"]).copy(), u16(host["v_state"]).copy()
    bt, sl = host["block_table"].numpy(), host["seq_lens"].numpy()
    oracle_mod.sconv_append(u16(host["k_new"]), ks, host["w_k"].numpy(), kc, bt, sl)
    oracle_mod.sconv_append(u16(host["v_new"]), vs, host["w_v"].numpy(), vc, bt, sl)
    # the GPU append (fp32 FMA chain, one bf16 rounding) against the oracle's
    # (exact sum, one bf16 rounding): within 1 bf16 ulp, or, where the four
    # tap products cancel, within the fp32 chain's rounding of the terms
    assert_append_close(u16(dev["k_cache"]), kc)
    assert_append_close(u16(dev["v_cache"]), vc)
    rng = np.random.default_rng(0)
    n = spec.chunk
    q = u16(host["q"]).reshape(spec.B, n, spec.Hq, 128)
    rows = np.array([[s, r, h] for s in range(spec.B)
                     for r in list(rng.integers(0, n, 6)) + [0, n - 1]
                     for h in rng.integers(0, spec.Hq, 2)], np.int32)
    ref, _ = oracle_mod.decode_mq_rows(q, kc, vc, bt, sl, host["bias"].numpy(), spec.window,
                                       spec.D_max, rows)
    got = out.cpu().reshape(spec.B, n, spec.Hq, 128)[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_parity(got, ref, "chunked workload sampled rows")
