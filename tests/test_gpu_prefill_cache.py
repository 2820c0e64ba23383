"""The prefill filling the paged cache and the sconv state in the same call,
on both execution paths (fused kernel; sconv append then paged prefill): bit
for bit what the sconv append writes for the same tokens, and a decode that
continues from it matches the oracle."""
import numpy as np
import pytest
import torch

from conftest import assert_parity, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import WORKLOADS, make_prefill, scaled

pytestmark = pytest.mark.gpu


def _setup(B, T, Hq, Hkv, W, D, seed, spare=2):
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], B=B, T=T, Hq=Hq, Hkv=Hkv, window=W,
                  D_max=D, seed=seed)
    t = make_prefill(spec)
    dev = {k: v.cuda() for k, v in t.items()}
    nb = (T + 127) // 128 + 1            # one block more than the prompt needs
    pool = B * nb + spare
    g = torch.Generator().manual_seed(seed)
    bt = torch.randperm(pool, generator=g)[:B * nb].reshape(B, nb).to(torch.int32).cuda()
    # stale cache contents: every slot the prompt does not cover must survive
    kc = torch.randn((pool, Hkv, 128, 128), generator=g).to(torch.bfloat16).cuda()
    vc = torch.randn((pool, Hkv, 128, 128), generator=g).to(torch.bfloat16).cuda()
    return spec, t, dev, bt, kc, vc


@pytest.mark.parametrize("B,T,Hq,Hkv,W", [
    (2, 1000, 16, 2, 300),   # G = 8: 4 heads x 128 rows per CTA pair, ragged last block
    (1, 700, 12, 2, 0),      # G = 6: 2 heads x 256 rows per CTA pair
    (2, 300, 6, 2, 100),     # G = 3: single-CTA kernel
    (1, 2, 8, 1, 0),         # T < 3: the state keeps zeros in front
    (1, 128, 8, 2, 0),       # exactly one block
    (3, 4096, 8, 1, 1024),   # several query blocks per sequence, window
])
@pytest.mark.parametrize("path", ["fused", "two_pass"])
def test_prefill_cache_equals_append(B, T, Hq, Hkv, W, path):
    need_gpu()
    spec, t, dev, bt, kc, vc = _setup(B, T, Hq, Hkv, W, 512, seed=T + Hq)
    kc2, vc2 = kc.clone(), vc.clone()
    C = Hkv * 128
    ks = torch.full((B, 3, C), 5.0, dtype=torch.bfloat16, device="cuda")   # overwritten
    vs = torch.full_like(ks, 5.0)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                           dev["bias"], window=W, status=status, k_cache=kc, v_cache=vc,
                           block_table=bt, k_state=ks, v_state=vs, path=path)
    plain = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                             dev["bias"], window=W, path=path)
    # the same tokens appended to empty sequences
    ks2 = torch.zeros((B, 3, C), dtype=torch.bfloat16, device="cuda")
    vs2 = torch.zeros_like(ks2)
    ink.sconv_kv(dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"], ks2, vs2, kc2, vc2, bt,
                 torch.full((B,), T, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(out.view(torch.int16), plain.view(torch.int16))
    assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
    assert torch.equal(ks.view(torch.int16), ks2.view(torch.int16))
    assert torch.equal(vs.view(torch.int16), vs2.view(torch.int16))


@pytest.mark.parametrize("path", ["fused", "two_pass"])
def test_decode_continues_from_prefill_cache(oracle_mod, path):
    """Serving order: prefill T tokens (filling cache and state), append one
    token with the sconv append, decode it; the oracle computes row T of the
    T+1-token sequence from the raw keys and values."""
    need_gpu()
    B, T, Hq, Hkv, W, D = 2, 900, 16, 2, 400, 700
    spec, t, dev, bt, kc, vc = _setup(B, T + 1, Hq, Hkv, W, D, seed=11)
    C = Hkv * 128
    ks = torch.zeros((B, 3, C), dtype=torch.bfloat16, device="cuda")
    vs = torch.zeros_like(ks)
    ink.attn_prefill(dev["q"][:, :T].contiguous(), dev["k_raw"][:, :T].contiguous(),
                     dev["v_raw"][:, :T].contiguous(), dev["w_k"], dev["w_v"], dev["bias"],
                     window=W, k_cache=kc, v_cache=vc, block_table=bt, k_state=ks, v_state=vs,
                     path=path)
    lens = torch.full((B,), T + 1, dtype=torch.int32, device="cuda")
    ink.sconv_kv(dev["k_raw"][:, T:].contiguous(), dev["v_raw"][:, T:].contiguous(), dev["w_k"],
                 dev["w_v"], ks, vs, kc, vc, bt, lens)
    dec = ink.attn_decode(dev["q"][:, T].contiguous(), kc, vc, bt, lens, dev["bias"], window=W)
    torch.cuda.synchronize()
    rows = np.array([[b, h, T] for b in range(B) for h in range(Hq)], np.int32)
    ref, _, _, _ = oracle_mod.prefill_rows(u16(t["q"]), u16(t["k_raw"]), u16(t["v_raw"]),
                                           t["w_k"].numpy(), t["w_v"].numpy(), t["bias"].numpy(),
                                           W, D, rows)
    assert_parity(dec.reshape(B * Hq, 128), ref, "decode after prefill cache fill")


@pytest.mark.parametrize("path", ["fused", "two_pass"])
def test_prefill_cache_bad_block_is_reported_and_skipped(path):
    """A block id outside the pool is reported and never written.  The fused
    kernel attends from its shared-memory tiles, so its rows stay right; the
    two-pass path reads the keys back from the cache, block 0 in place of the
    bad one, so only the rows that never see that block are checked."""
    need_gpu()
    B, T, Hq, Hkv = 1, 300, 8, 1
    spec, t, dev, bt, kc, vc = _setup(B, T, Hq, Hkv, 0, 300, seed=5)
    bt[0, 1] = kc.shape[0] + 7            # outside the pool: never dereferenced
    before = kc.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                           dev["bias"], status=status, k_cache=kc, v_cache=vc, block_table=bt,
                           path=path)
    plain = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                             dev["bias"], path=path)
    torch.cuda.synchronize()
    assert status.item() & 2              # INKLING_STATUS_BAD_BLOCK
    rows = slice(None) if path == "fused" else slice(0, 128)   # rows 0..127 see block 0 only
    assert torch.equal(out[:, rows].view(torch.int16), plain[:, rows].view(torch.int16))
    # the valid blocks were written, the pool is otherwise unchanged
    assert not torch.equal(kc[bt[0, 0]], before[bt[0, 0]])
    untouched = [i for i in range(kc.shape[0]) if i not in (int(bt[0, 0]), int(bt[0, 2]))]
    assert torch.equal(kc[untouched].view(torch.int16), before[untouched].view(torch.int16))


def test_prefill_cache_argument_errors():
    need_gpu()
    spec, t, dev, bt, kc, vc = _setup(1, 300, 8, 1, 0, 300, seed=6)
    args = (dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"], dev["bias"])
    with pytest.raises(ValueError):
        ink.attn_prefill(*args, k_cache=kc, block_table=bt)            # v_cache missing
    with pytest.raises(ink.InklingError):
        ink.attn_prefill(*args, k_cache=kc, v_cache=vc, block_table=bt[:, :2])  # 256 < 300
