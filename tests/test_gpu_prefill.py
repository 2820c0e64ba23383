"""tcgen05 prefill on the GPU against the oracle, plus invariants, on both
execution paths: the fused kernel (sconv applied to each key/value tile in
shared memory) and the two-pass one (sconv written once in the paged layout,
then the paged prefill kernel)."""
import numpy as np
import pytest
import torch

from conftest import assert_parity, need_gpu, u16
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import WORKLOADS, make_prefill, scaled

pytestmark = pytest.mark.gpu
PATHS = ("fused", "two_pass")


def _run(t, window, with_lse=True, path="auto"):
    dev = {k: v.cuda() for k, v in t.items()}
    B, T, Hq, _ = dev["q"].shape
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda") if with_lse else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                           dev["bias"], window=window, lse=lse, status=status, path=path)
    torch.cuda.synchronize()
    assert status.item() == 0, f"status {status.item()}"
    return out, lse


def _oracle_all(oracle_mod, t, window):
    out, lse, _, _ = oracle_mod.prefill_rows(u16(t["q"]), u16(t["k_raw"]), u16(t["v_raw"]),
                                             t["w_k"].numpy(), t["w_v"].numpy(),
                                             t["bias"].numpy(), window, t["bias"].shape[1] - 1)
    return out, lse


def test_prefill_tiny_workload_all_rows(oracle_mod):
    need_gpu()
    spec = WORKLOADS["prefill_tiny_b1_t256"]
    t = make_prefill(spec)
    ref, ref_lse = _oracle_all(oracle_mod, t, spec.window)
    for path in PATHS:
        out, lse = _run(t, spec.window, path=path)
        assert_parity(out, ref, f"{spec.name} {path}")
        got_lse = lse.permute(0, 2, 1).cpu().numpy().reshape(-1)   # [B, T, Hq] order
        np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=2e-3)


@pytest.mark.parametrize("B,T,Hq,Hkv,W,D_max", [
    (1, 1, 8, 1, 0, 16),         # a single token
    (1, 129, 8, 1, 0, 256),      # one row past a tile
    (2, 300, 8, 2, 0, 64),       # ragged tail, GQA 4, clip inside the band
    (1, 700, 4, 1, 100, 1000),   # window narrower than a tile
    (1, 640, 8, 8, 128, 128),    # window exactly one tile, G = 1
    (1, 1000, 16, 2, 300, 50),   # window + clip, ragged
    (1, 520, 8, 1, 1, 8),        # window of one key (self only)
    (3, 257, 8, 4, 256, 300),    # query block boundary + 1
    (1, 600, 12, 2, 200, 300),   # G = 6: two heads x 256 rows per CTA pair
    (2, 400, 12, 3, 0, 400),     # G = 4, three kv heads: four heads x 128 rows per pair
    (2, 130, 6, 2, 0, 200),      # G = 3 (single-CTA fused kernel), 2 blocks, 2 rows past one
])
def test_prefill_ragged_and_masks(oracle_mod, B, T, Hq, Hkv, W, D_max):
    need_gpu()
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], B=B, T=T, Hq=Hq, Hkv=Hkv, window=W,
                  D_max=D_max, seed=T + W)
    t = make_prefill(spec)
    ref, ref_lse = _oracle_all(oracle_mod, t, W)
    got = {}
    for path in PATHS:
        out, lse = _run(t, W, path=path)
        assert_parity(out, ref, f"B{B} T{T} Hq{Hq} Hkv{Hkv} W{W} D{D_max} {path}")
        got_lse = lse.permute(0, 2, 1).cpu().numpy().reshape(-1)
        np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=2e-3)
        got[path] = (out, lse)
    # the two paths give the same bits (same MMA order and softmax code)
    assert torch.equal(got["fused"][0].view(torch.int16), got["two_pass"][0].view(torch.int16))
    assert torch.equal(got["fused"][1], got["two_pass"][1])


@pytest.mark.parametrize("B,T,Hq,Hkv,W", [
    (1, 2560, 32, 4, 0),      # 160 CTA pairs: more than fit on the GPU at once
    (2, 2500, 32, 4, 1000),   # 320 pairs, ragged tail, window not a multiple of a tile
    (1, 2900, 24, 4, 700),    # G = 6 (two heads x 256 rows per pair), 132 pairs, ragged
])
def test_prefill_several_waves_all_rows(oracle_mod, B, T, Hq, Hkv, W):
    """More (head pair, query block) CTA pairs than fit on the GPU at once, with
    full and partial (window-edge, diagonal, ragged-tail) tiles; every row and
    its log-sum-exp are compared."""
    need_gpu()
    spec = scaled(WORKLOADS["prefill_swa_b4_t8192"], B=B, T=T, Hq=Hq, Hkv=Hkv, window=W,
                  D_max=3000, seed=11 + W)
    t = make_prefill(spec)
    ref, ref_lse = _oracle_all(oracle_mod, t, W)
    got = {}
    for path in PATHS:
        out, lse = _run(t, W, path=path)
        assert_parity(out, ref, f"B{B} T{T} Hq{Hq} Hkv{Hkv} W{W} {path}")
        got_lse = lse.permute(0, 2, 1).cpu().numpy().reshape(-1)
        np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=2e-3)
        got[path] = (out, lse)
    assert torch.equal(got["fused"][0].view(torch.int16), got["two_pass"][0].view(torch.int16))
    assert torch.equal(got["fused"][1], got["two_pass"][1])


@pytest.mark.parametrize("path", PATHS)
def test_prefill_window_at_least_T_equals_full(path):
    need_gpu()
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], T=600, Hq=8, Hkv=2, D_max=700, seed=5)
    t = make_prefill(spec)
    full, _ = _run(t, 0, path=path)
    win, _ = _run(t, 600, path=path)
    assert torch.equal(full, win)


@pytest.mark.parametrize("B,T,two", [(1, 2047, False), (1, 2048, True), (4, 511, False),
                                     (4, 512, True), (2, 1000, False)])
def test_prefill_auto_path_follows_the_thresholds(B, T, two):
    """The automatic path runs the two passes when B*T >= 2048 tokens and
    T >= 512, and fuses otherwise: the library asks for a workspace only then,
    and a workspace passed then is written by the first pass.  The two paths
    give the same bits: the same MMA order and softmax code over the same
    post-sconv keys and values."""
    need_gpu()
    Hq, Hkv = 16, 2
    spec = scaled(WORKLOADS["prefill_swa_b4_t8192"], B=B, T=T, Hq=Hq, Hkv=Hkv, window=1000,
                  D_max=3000, seed=T + B)
    t = make_prefill(spec)
    dev = {k: v.cuda() for k, v in t.items()}
    need = ink.prefill_workspace_bytes(B, T, Hq, Hkv)
    assert (need > 0) == two
    ws = torch.full((max(need, 16),), 0xff, dtype=torch.uint8, device="cuda")
    lse = torch.empty((B, Hq, T), dtype=torch.float32, device="cuda")
    auto = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                            dev["bias"], window=1000, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    assert bool((ws != 0xff).any()) == two
    for path in PATHS:
        out, lse2 = _run(t, 1000, path=path)
        assert torch.equal(auto.view(torch.int16), out.view(torch.int16)), path
        assert torch.equal(lse, lse2), path


def test_prefill_two_pass_uses_the_given_workspace(oracle_mod):
    """With a workspace passed in, the two-pass path writes the post-sconv
    keys/values there, in the paged layout (sequence b on blocks b*nb ...),
    bit for bit what the sconv append writes for the same tokens, and zeroes
    the slots past the end of each sequence's last block: a workspace full of
    NaN bits gives the oracle's rows."""
    need_gpu()
    B, T, Hq, Hkv = 2, 300, 8, 2
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], B=B, T=T, Hq=Hq, Hkv=Hkv, D_max=300, seed=9)
    t = make_prefill(spec)
    dev = {k: v.cuda() for k, v in t.items()}
    nb = (T + 127) // 128
    need = ink.prefill_workspace_bytes(B, T, Hq, Hkv, path="two_pass")
    assert need == 2 * B * nb * Hkv * 128 * 128 * 2
    ws = torch.full((need + 64,), 0xff, dtype=torch.uint8, device="cuda")   # bf16 NaN bits
    out = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                           dev["bias"], path="two_pass", workspace=ws)
    kc = torch.zeros((B * nb, Hkv, 128, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    st = torch.zeros((B, 3, Hkv * 128), dtype=torch.bfloat16, device="cuda")
    st2 = torch.zeros_like(st)
    bt = torch.arange(B * nb, dtype=torch.int32, device="cuda").reshape(B, nb)
    ink.sconv_kv(dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"], st, st2, kc, vc, bt,
                 torch.full((B,), T, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    half = need // 2
    got_k = ws[:half].view(torch.bfloat16).reshape(kc.shape)
    got_v = ws[half:need].view(torch.bfloat16).reshape(vc.shape)
    for b in range(B):
        for blk in range(nb):
            n = min(128, T - blk * 128)
            i = b * nb + blk
            assert torch.equal(got_k[i, :, :n].view(torch.int16), kc[i, :, :n].view(torch.int16))
            assert torch.equal(got_v[i, :, :n].view(torch.int16), vc[i, :, :n].view(torch.int16))
            assert (got_k[i, :, n:].view(torch.int16) == 0).all()
            assert (got_v[i, :, n:].view(torch.int16) == 0).all()
    assert (ws[need:] == 0xff).all()   # nothing past the workspace size
    ref, _, _, _ = oracle_mod.prefill_rows(u16(t["q"]), u16(t["k_raw"]), u16(t["v_raw"]),
                                           t["w_k"].numpy(), t["w_v"].numpy(), t["bias"].numpy(),
                                           0, 300)
    assert_parity(out, ref, "two-pass over a NaN-filled workspace")
    again = ink.attn_prefill(dev["q"], dev["k_raw"], dev["v_raw"], dev["w_k"], dev["w_v"],
                             dev["bias"], path="two_pass")   # scratch allocated by the binding
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), again.view(torch.int16))


@pytest.mark.parametrize("path", PATHS)
def test_prefill_empty_batch_is_noop(path):
    need_gpu()
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], B=1, T=16)
    t = make_prefill(spec)
    dev = {k: v.cuda() for k, v in t.items()}
    out = torch.full((0, 16, 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    ink.attn_prefill(dev["q"][:0], dev["k_raw"][:0], dev["v_raw"][:0], dev["w_k"], dev["w_v"],
                     dev["bias"], out=out, path=path)
    torch.cuda.synchronize()


def test_prefill_last_row_equals_decode(oracle_mod):
    """Prefill row T-1 equals decode at length T over the cache that
    sconv_kv builds from the same raw keys and values (streaming continuity)."""
    need_gpu()
    T, Hq, Hkv, W, D = 1000, 16, 2, 300, 512
    spec = scaled(WORKLOADS["prefill_tiny_b1_t256"], T=T, Hq=Hq, Hkv=Hkv, window=W, D_max=D,
                  seed=3)
    t = make_prefill(spec)
    out, _ = _run(t, W)
    dev = {k: v.cuda() for k, v in t.items()}
    nb = (T + 127) // 128
    kc = torch.zeros((nb + 2, Hkv, 128, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    bt = torch.arange(2, nb + 2, dtype=torch.int32, device="cuda")[None]
    ks = torch.zeros((1, 3, Hkv * 128), dtype=torch.bfloat16, device="cuda")
    vs = torch.zeros_like(ks)
    done = 0
    while done < T:
        n = min(64, T - done)
        ink.sconv_kv(dev["k_raw"][:, done:done + n].contiguous(),
                     dev["v_raw"][:, done:done + n].contiguous(), dev["w_k"], dev["w_v"], ks, vs,
                     kc, vc, bt, torch.tensor([done + n], dtype=torch.int32, device="cuda"))
        done += n
    dec = ink.attn_decode(dev["q"][:, T - 1].contiguous(), kc, vc, bt,
                          torch.tensor([T], dtype=torch.int32, device="cuda"), dev["bias"],
                          window=W, num_splits=3)
    torch.cuda.synchronize()
    assert (dec.float() - out[:, T - 1].float()).abs().max().item() < 2e-2
    rows = np.array([[0, h, T - 1] for h in range(Hq)], np.int32)
    ref, _, _, _ = oracle_mod.prefill_rows(u16(t["q"]), u16(t["k_raw"]), u16(t["v_raw"]),
                                           t["w_k"].numpy(), t["w_v"].numpy(), t["bias"].numpy(),
                                           W, D, rows)
    assert_parity(dec[0], ref, "decode vs oracle")


def _sample_rows(spec, rng, per_head):
    """Stratified rows of every (batch, head): the first 128 rows, the window
    edge W-1 .. W+128 (sliding window only), the last 128 rows, and
    `per_head` random rows (the first query blocks, the rows where keys start
    to leave the window, the diagonal tiles of the last query blocks, and
    rows anywhere)."""
    T, W = spec.T, spec.window
    fixed = list(range(0, min(128, T)))
    if W > 0:
        fixed += list(range(max(0, W - 1), min(T, W + 129)))
    fixed += list(range(max(0, T - 128), T))
    fixed = sorted(set(fixed))
    rows = []
    for b in range(spec.B):
        for h in range(spec.Hq):
            pick = fixed + list(rng.integers(0, T, size=per_head))
            rows += [(b, h, i) for i in pick]
    return np.array(rows, np.int32)


@pytest.mark.parametrize("name,per_head", [("prefill_swa_b4_t8192", 256),
                                           ("prefill_full_b1_t32768", 256)])
def test_prefill_full_size_sampled_rows(oracle_mod, name, per_head):
    """The benchmark workloads at full size, in the benchmark's launch
    configuration (the automatic path, two-pass at these lengths) and on the
    fused kernel; the oracle computes a sample of rows of every (batch, head),
    with their log-sum-exp."""
    need_gpu()
    spec = WORKLOADS[name]
    t = make_prefill(spec, device="cuda")
    rows = _sample_rows(spec, np.random.default_rng(0), per_head)
    ref, ref_lse, _, _ = oracle_mod.prefill_rows(u16(t["q"]), u16(t["k_raw"]), u16(t["v_raw"]),
                                                 t["w_k"].cpu().numpy(), t["w_v"].cpu().numpy(),
                                                 t["bias"].cpu().numpy(), spec.window,
                                                 spec.D_max, rows)
    r = torch.from_numpy(rows).long().cuda()
    first = None
    for path in ("auto", "fused"):
        lse = torch.empty((spec.B, spec.Hq, spec.T), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = ink.attn_prefill(t["q"], t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], t["bias"],
                               window=spec.window, status=status, lse=lse, path=path)
        torch.cuda.synchronize()
        assert status.item() == 0
        got = out[r[:, 0], r[:, 2], r[:, 1]].float().cpu().numpy()
        assert_parity(got, ref, f"{name} {path}")
        got_lse = lse[r[:, 0], r[:, 1], r[:, 2]].cpu().numpy()
        np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=2e-3)
        if first is None:
            first = (out, lse)
        else:   # the two paths give the same bits at full size too
            assert torch.equal(first[0].view(torch.int16), out.view(torch.int16))
            assert torch.equal(first[1], lse)
