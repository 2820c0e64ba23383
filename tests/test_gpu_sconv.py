"""sconv_kv on the GPU against the oracle's decode-side append."""
import numpy as np
import pytest
import torch

from conftest import assert_append_close, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import BLOCK

pytestmark = pytest.mark.gpu


def _setup(S, Hkv, lens, n_new, seed, dyadic=False, extra=3):
    g = torch.Generator().manual_seed(seed)
    d = 128
    C = Hkv * d
    if dyadic:
        mk = lambda *sh: torch.randint(-8, 9, sh, generator=g).to(torch.bfloat16)
        w_k = (torch.randint(-4, 5, (C, 4), generator=g) / 4).float()
        w_v = (torch.randint(-4, 5, (C, 4), generator=g) / 4).float()
    else:
        mk = lambda *sh: torch.randn(sh, generator=g).to(torch.bfloat16)
        w_k = torch.randn((C, 4), generator=g) * 0.5
        w_v = torch.randn((C, 4), generator=g) * 0.5
    k_new, v_new = mk(S, n_new, Hkv, d), mk(S, n_new, Hkv, d)
    k_state, v_state = mk(S, 3, C), mk(S, 3, C)
    nb = [(L + BLOCK - 1) // BLOCK for L in lens]
    total = sum(nb) + extra
    perm = torch.randperm(total, generator=g).to(torch.int32)
    max_blocks = max(nb)
    bt = torch.zeros((S, max_blocks), dtype=torch.int32)
    off = 0
    for s in range(S):
        bt[s, :nb[s]] = perm[off:off + nb[s]]
        off += nb[s]
    k_cache, v_cache = mk(total, Hkv, BLOCK, d), mk(total, Hkv, BLOCK, d)
    return dict(k_new=k_new, v_new=v_new, w_k=w_k, w_v=w_v, k_state=k_state, v_state=v_state,
                k_cache=k_cache, v_cache=v_cache, block_table=bt,
                seq_lens=torch.tensor(lens, dtype=torch.int32))


def _run_both(oracle_mod, t):
    dev = {k: v.cuda() for k, v in t.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ink.sconv_kv(**dev, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = {}
    for which in ("k", "v"):
        state = u16(t[f"{which}_state"]).copy()
        cache = u16(t[f"{which}_cache"]).copy()
        oracle_mod.sconv_append(u16(t[f"{which}_new"]), state, t[f"w_{which}"].numpy(), cache,
                                t["block_table"].numpy(), t["seq_lens"].numpy())
        ref[which] = (state, cache)
    return dev, ref


@pytest.mark.parametrize("n_new,lens", [(1, [1, 128, 129, 5000, 300]), (2, [2, 3, 400]),
                                        (3, [3, 130, 256]), (7, [7, 200, 1000]),
                                        (33, [33, 34, 300]), (64, [64, 127, 4096]),
                                        (1029, [1029, 1300, 4096])])
def test_sconv_kv_matches_oracle(oracle_mod, n_new, lens):
    need_gpu()
    t = _setup(len(lens), 2, lens, n_new, seed=n_new)
    dev, ref = _run_both(oracle_mod, t)
    for which in ("k", "v"):
        st_ref, cache_ref = ref[which]
        # the state holds raw bf16 tokens: exact
        assert np.array_equal(u16(dev[f"{which}_state"]), st_ref)
        got = u16(dev[f"{which}_cache"]).view(np.int16).astype(np.int32)
        exp = cache_ref.view(np.int16).astype(np.int32)
        # fp32 FMA chain vs one rounding of the exact sum: rarely different,
        # within 1 bf16 ulp or (cancelling taps) the chain's fp32 rounding
        frac = assert_append_close(u16(dev[f"{which}_cache"]), cache_ref)
        assert frac < 2e-3, which
        # untouched slots are bit-identical (paging is index work: exact)
        untouched = np.ones(exp.shape, bool)
        bt = t["block_table"].numpy()
        for s, L in enumerate(lens):
            for pos in range(L - n_new, L):
                untouched[bt[s, pos // 128], :, pos % 128, :] = False
        assert np.array_equal(got[untouched], exp[untouched])


def test_sconv_kv_exact_on_dyadic_inputs(oracle_mod):
    need_gpu()
    lens = [5, 128, 129, 777]
    t = _setup(len(lens), 3, lens, 5, seed=11, dyadic=True)
    dev, ref = _run_both(oracle_mod, t)
    for which in ("k", "v"):
        assert np.array_equal(u16(dev[f"{which}_state"]), ref[which][0])
        assert np.array_equal(u16(dev[f"{which}_cache"]), ref[which][1])


def test_sconv_kv_reports_bad_block_and_length():
    need_gpu()
    t = _setup(2, 1, [10, 200], 1, seed=5)
    t["block_table"][1, 1] = 10_000          # out of the pool
    dev = {k: v.cuda() for k, v in t.items()}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ink.sconv_kv(**dev, status=status)
    torch.cuda.synchronize()
    assert status.item() & ink.binding.STATUS_BAD_BLOCK
    dev["seq_lens"][0] = 0                   # shorter than n_new
    status.zero_()
    ink.sconv_kv(**dev, status=status)
    torch.cuda.synchronize()
    assert status.item() & ink.binding.STATUS_BAD_LENGTH
