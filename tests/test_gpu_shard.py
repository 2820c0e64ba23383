"""The layer sharded over kv heads (tensor parallelism): a call of the library
on one shard of kv heads, with the matching query heads, taps, sconv states,
cache slices and bias rows, equals that shard's slice of the call on the whole
layer, bit for bit.  The sconv is depthwise, so its channels shard with the kv
heads and no exchange is needed inside the layer (vLLM Recipes
"thinkingmachines/Inkling", Overview "Short convolution" and Performance:
sconv-aware sharding, each rank keeping only its channel shard of the sconv
cache)."""
import pytest
import torch

from conftest import need_gpu
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import WORKLOADS, make_decode, make_prefill, scaled

pytestmark = pytest.mark.gpu


def _heads(N, r, Hq, Hkv):
    """(query-head slice, kv-head slice, channel slice) of shard r of N."""
    hk = Hkv // N
    hq = Hq // N
    return (slice(r * hq, (r + 1) * hq), slice(r * hk, (r + 1) * hk),
            slice(r * hk * 128, (r + 1) * hk * 128))


@pytest.mark.parametrize("N,window", [(2, 300), (4, 0)])
def test_prefill_kv_head_shard_equals_slice(N, window):
    need_gpu()
    spec = scaled(WORKLOADS["prefill_swa_b4_t8192"], B=2, T=700, Hq=32, Hkv=4, window=window,
                  D_max=512, seed=31)
    t = {k: v.cuda() for k, v in make_prefill(spec).items()}
    full = ink.attn_prefill(t["q"], t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], t["bias"],
                            window=window)
    for r in range(N):
        qh, kh, ch = _heads(N, r, spec.Hq, spec.Hkv)
        out = ink.attn_prefill(t["q"][:, :, qh].contiguous(), t["k_raw"][:, :, kh].contiguous(),
                               t["v_raw"][:, :, kh].contiguous(), t["w_k"][ch].contiguous(),
                               t["w_v"][ch].contiguous(), t["bias"][qh].contiguous(),
                               window=window)
        torch.cuda.synchronize()
        assert torch.equal(out, full[:, :, qh]), f"shard {r} of {N}"


@pytest.mark.parametrize("q_len", [1, 4])
def test_append_and_decode_kv_head_shard_equals_slice(q_len):
    need_gpu()
    N = 2
    spec = scaled(WORKLOADS["decode_swa_s64"], S=5, L_min=200, L_max=9000, window=4096,
                  n_new=q_len, seed=32)
    t = make_decode(spec, device="cuda")
    full = {k: v.clone() for k, v in t.items()}
    ink.sconv_kv(full["k_new"], full["v_new"], full["w_k"], full["w_v"], full["k_state"],
                 full["v_state"], full["k_cache"], full["v_cache"], full["block_table"],
                 full["seq_lens"])
    out_full = ink.attn_decode(full["q"], full["k_cache"], full["v_cache"], full["block_table"],
                               full["seq_lens"], full["bias"], window=spec.window, num_splits=3)
    hd = 2 if q_len > 1 else 1  # head axis of q
    for r in range(N):
        qh, kh, ch = _heads(N, r, spec.Hq, spec.Hkv)
        sh = {k: v.clone() for k, v in t.items()}
        kc = sh["k_cache"][:, kh].contiguous()
        vc = sh["v_cache"][:, kh].contiguous()
        ks = sh["k_state"][:, :, ch].contiguous()
        vs = sh["v_state"][:, :, ch].contiguous()
        ink.sconv_kv(sh["k_new"][:, :, kh].contiguous(), sh["v_new"][:, :, kh].contiguous(),
                     sh["w_k"][ch].contiguous(), sh["w_v"][ch].contiguous(), ks, vs, kc, vc,
                     sh["block_table"], sh["seq_lens"])
        q = sh["q"][:, :, qh] if hd == 2 else sh["q"][:, qh]
        out = ink.attn_decode(q.contiguous(), kc, vc, sh["block_table"], sh["seq_lens"],
                              sh["bias"][qh].contiguous(), window=spec.window, num_splits=3)
        torch.cuda.synchronize()
        assert torch.equal(kc, full["k_cache"][:, kh]) and torch.equal(vc, full["v_cache"][:, kh])
        assert torch.equal(ks, full["k_state"][:, :, ch]) and torch.equal(vs, full["v_state"][:, :, ch])
        ref = out_full[:, :, qh] if hd == 2 else out_full[:, qh]
        assert torch.equal(out, ref), f"shard {r} of {N}"


def _parts(N, B, T, C, seed):
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn(B, T, C, generator=g).to(torch.bfloat16).cuda() for _ in range(N)]
    w = (torch.randn(C, 4, generator=g) * 0.5).cuda()
    state = torch.randn(B, 3, C, generator=g).to(torch.bfloat16).cuda()
    return xs, w, state


@pytest.mark.parametrize("N,T,with_state", [(1, 300, True), (2, 300, True), (4, 70, False),
                                            (8, 129, True), (2, 2, True)])
def test_sharded_output_sconv_one_kernel_over_all_ranks_buffers(oracle_mod, N, T, with_state):
    """The fused reduce-scatter / sconv / all-gather kernel, with the N ranks'
    buffers emulated on one GPU (each rank's call reads every rank's partial
    sum and writes every rank's output): after all N calls every output equals
    the unsharded output sconv of the summed input (fp32 sum in rank order,
    one bf16 rounding), bit for bit, and matches the oracle; the state shards
    equal the slices of the unsharded state; a second round continues from
    them."""
    need_gpu()
    from conftest import assert_append_close, u16
    from relative_bias_sliding_b200.sharded import channel_shard
    B, C = 2, 1024
    xs, w, state = _parts(N, B, T, C, seed=40 + N)
    acc = xs[0].float()
    for x in xs[1:]:
        acc = acc + x.float()
    s = acc.to(torch.bfloat16)
    full_state = state.clone() if with_state else None
    shards = [state[:, :, channel_shard(C, N, r)].clone() if with_state else None
              for r in range(N)]
    for rnd in range(2):
        ys = [torch.full_like(xs[0], float("nan")) for _ in range(N)]
        for r in range(N):
            ink.sconv_out_sharded(xs, w, ys, r, state=shards[r])
        ref = ink.sconv_out(s, w, full_state)
        torch.cuda.synchronize()
        for r in range(N):
            assert torch.equal(ys[r], ref), f"round {rnd}: output of rank {r}"
            if with_state:
                assert torch.equal(shards[r], full_state[:, :, channel_shard(C, N, r)])
        if rnd == 0:
            hist = None if not with_state else u16(state)
            exp = oracle_mod.sconv(u16(s), w.cpu().numpy(), hist)
            assert_append_close(u16(ys[0]), exp)
