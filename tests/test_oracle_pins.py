"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties the oracle to something it does not compute itself: hand-derived
values (tests/golden), IEEE rounding rules, numpy's convolution, torch's
scaled-dot-product attention in fp64, closed forms and invariants of softmax.
Together they are chosen so that a dropped term, a wrong sign or index
(i-j vs j-i), a transposed operand, a wrong GQA map or a wrong clip fails at
least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import u16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def bf16_bits(x):
    """numpy fp32 -> bf16 bits via the textbook round-half-to-even bit trick
    (exact for fp32 inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def f64(bits):
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_bf16(shape, std=1.0):
    return bf16_bits(rng.standard_normal(shape).astype(np.float32) * std)


# ---------------------------------------------------------------- rounding --

def test_bf16_rounding_golden(oracle_mod):
    n = 0
    with open(os.path.join(GOLDEN, "bf16_rne.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            val, exp = line.split()[:2]
            assert oracle_mod.f64_to_bf16(float.fromhex(val)) == int(exp, 16), line
            n += 1
    assert n >= 14


def test_bf16_rounding_matches_bit_trick_on_fp32(oracle_mod):
    xs = rng.standard_normal(4000).astype(np.float32) * np.float32(3.0)
    xs = np.concatenate([xs, np.float32([1e-39, -3e-40, 1e30, 65504.0])])
    exp = bf16_bits(xs)
    got = np.array([oracle_mod.f64_to_bf16(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, exp)
    back = np.array([oracle_mod.bf16_to_f64(int(b)) for b in exp[:50]])
    assert np.array_equal(back, f64(exp[:50]))


# ------------------------------------------------------------------- sconv --

def test_sconv_matches_numpy_convolve(oracle_mod):
    B, T, C = 2, 37, 16
    x = rand_bf16((B, T, C))
    w = (rng.standard_normal((C, 4)) * 0.5).astype(np.float32)
    y = oracle_mod.sconv(x, w)
    ref = np.empty((B, T, C))
    for b in range(B):
        for c in range(C):
            ref[b, :, c] = np.convolve(f64(x[b, :, c]), w[c].astype(np.float64))[:T]
    got = f64(y)
    # one rounding to bf16: within half a bf16 ulp of the exact sum
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    assert np.all(np.abs(got - ref) <= 0.5 * ulp * (1 + 1e-12))


def test_sconv_exact_on_dyadic_inputs(oracle_mod):
    # small integers and dyadic taps: every sum is exact in bf16
    B, T, C = 1, 20, 8
    xi = rng.integers(-8, 9, size=(B, T, C)).astype(np.float32)
    w = rng.integers(-4, 5, size=(C, 4)).astype(np.float32) / 4
    y = oracle_mod.sconv(bf16_bits(xi), w)
    ref = np.empty((B, T, C))
    for c in range(C):
        ref[0, :, c] = np.convolve(xi[0, :, c].astype(np.float64), w[c].astype(np.float64))[:T]
    assert np.array_equal(y, bf16_bits(ref.astype(np.float32)))


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_sconv_delta_taps_shift(oracle_mod, tap):
    B, T, C = 2, 11, 4
    x = rand_bf16((B, T, C))
    w = np.zeros((C, 4), np.float32)
    w[:, tap] = 1.0
    y = oracle_mod.sconv(x, w)
    exp = np.zeros_like(x)
    exp[:, tap:, :] = x[:, : T - tap, :]
    assert np.array_equal(y, exp)


def test_sconv_streaming_equals_batch(oracle_mod):
    # feeding one token at a time with the rolling raw-token state reproduces
    # the whole-sequence convolution (the state acts as a 3-token sliding cache)
    B, T, C = 2, 9, 6
    x = rand_bf16((B, T, C))
    w = (rng.standard_normal((C, 4)) * 0.5).astype(np.float32)
    batch = oracle_mod.sconv(x, w)
    hist = np.zeros((B, 3, C), np.uint16)
    for t in range(T):
        yt = oracle_mod.sconv(x[:, t:t + 1, :], w, hist)
        assert np.array_equal(yt[:, 0, :], batch[:, t, :])
        hist = np.concatenate([hist[:, 1:, :], x[:, t:t + 1, :]], axis=1)


def test_sconv_append_paged_equals_batch(oracle_mod):
    S, Hkv, d, T = 2, 2, 8, 300
    C = Hkv * d
    x = rand_bf16((S, T, Hkv, d))
    w = (rng.standard_normal((C, 4)) * 0.5).astype(np.float32)
    batch = oracle_mod.sconv(x.reshape(S, T, C), w).reshape(S, T, Hkv, d)
    nb = (T + 127) // 128
    perm = rng.permutation(S * nb).astype(np.int32)
    bt = perm.reshape(S, nb)
    cache = np.zeros((S * nb, Hkv, 128, d), np.uint16)
    state = np.zeros((S, 3, C), np.uint16)
    done = 0
    for n_new in [5, 1, 2, 130, 1, 161]:
        lens = np.full(S, done + n_new, np.int32)
        oracle_mod.sconv_append(np.ascontiguousarray(x[:, done:done + n_new]), state, w, cache,
                                bt, lens)
        done += n_new
    assert done == T
    for s in range(S):
        for j in range(T):
            assert np.array_equal(cache[bt[s, j // 128], :, j % 128, :], batch[s, j])
    assert np.array_equal(state, x[:, T - 3:].reshape(S, 3, C))


# --------------------------------------------------------------- attention --

def sdpa_reference(q, kc, vc, bias, window, D_max):
    """torch fp64 scaled_dot_product_attention with an additive float mask
    bias[h, min(i-j, D_max)] (-inf outside the causal band / window) and the
    kv heads repeated G times (contiguous grouping)."""
    B, T, Hq, d = q.shape
    Hkv = kc.shape[2]
    G = Hq // Hkv
    Q = torch.from_numpy(f64(q)).permute(0, 2, 1, 3)
    K = torch.from_numpy(f64(kc)).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    V = torch.from_numpy(f64(vc)).permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    dist = i - j
    allowed = dist >= 0
    if window > 0:
        allowed &= dist < window
    idx = dist.clamp(min=0, max=D_max)
    bt = torch.from_numpy(bias.astype(np.float64))
    mask = bt[:, idx]                                    # [Hq, T, T]
    mask = torch.where(allowed[None], mask, torch.tensor(-math.inf, dtype=torch.float64))
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask[None])
    scores = (Q @ K.transpose(-1, -2)) / math.sqrt(d) + mask[None]
    lse = torch.logsumexp(scores, dim=-1)                # [B, Hq, T]
    return out.permute(0, 2, 1, 3).numpy(), lse.permute(0, 2, 1).numpy()


def identity_taps(C):
    w = np.zeros((C, 4), np.float32)
    w[:, 0] = 1.0
    return w


@pytest.mark.parametrize("B,T,Hq,Hkv,window,D_max", [
    (1, 40, 4, 1, 0, 64),      # full causal, no clip reached
    (2, 33, 8, 2, 7, 64),      # sliding window, GQA group 4
    (1, 50, 4, 2, 0, 9),       # distance clip at D_max < T
    (1, 29, 6, 3, 5, 3),       # window and clip together
])
def test_attention_matches_torch_sdpa(oracle_mod, B, T, Hq, Hkv, window, D_max):
    d = 128
    q = rand_bf16((B, T, Hq, d))
    k = rand_bf16((B, T, Hkv, d))
    v = rand_bf16((B, T, Hkv, d))
    bias = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    C = Hkv * d
    out, lse, kc, vc = oracle_mod.prefill_rows(q, k, v, identity_taps(C), identity_taps(C),
                                               bias, window, D_max)
    assert np.array_equal(kc, k) and np.array_equal(vc, v)
    ref, ref_lse = sdpa_reference(q, k, v, bias, window, D_max)
    np.testing.assert_allclose(out.reshape(B, T, Hq, d), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(B, T, Hq), ref_lse, rtol=0, atol=1e-12)


def test_sconv_then_attention_matches_library_chain(oracle_mod):
    # non-trivial taps: numpy convolution -> bf16 -> torch SDPA
    B, T, Hq, Hkv, d, W, D_max = 1, 24, 4, 2, 128, 6, 30
    C = Hkv * d
    q = rand_bf16((B, T, Hq, d))
    k = rand_bf16((B, T, Hkv, d))
    v = rand_bf16((B, T, Hkv, d))
    wk = (rng.integers(-4, 5, size=(C, 4)) / 8).astype(np.float32)
    wv = (rng.integers(-4, 5, size=(C, 4)) / 8).astype(np.float32)
    bias = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    out, lse, kc, vc = oracle_mod.prefill_rows(q, k, v, wk, wv, bias, W, D_max)

    def conv(x, w):
        xf = f64(x).reshape(B, T, C)
        y = np.empty_like(xf)
        for c in range(C):
            y[0, :, c] = np.convolve(xf[0, :, c], w[c].astype(np.float64))[:T]
        return y.reshape(B, T, Hkv, d)

    kref, vref = conv(k, wk), conv(v, wv)
    # each post-sconv value is the exact sum rounded once to bf16
    for got, ref in ((kc, kref), (vc, vref)):
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
        assert np.all(np.abs(f64(got) - ref) <= 0.5 * ulp * (1 + 1e-12))
    r, _ = sdpa_reference(q, kc, vc, bias, W, D_max)
    np.testing.assert_allclose(out.reshape(B, T, Hq, d), r, rtol=0, atol=1e-12)


def test_zero_bias_is_plain_causal_attention(oracle_mod):
    B, T, Hq, Hkv, d = 1, 31, 4, 2, 128
    q, k, v = rand_bf16((B, T, Hq, d)), rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    bias = np.zeros((Hq, 65), np.float32)
    C = Hkv * d
    out, _, _, _ = oracle_mod.prefill_rows(q, k, v, identity_taps(C), identity_taps(C), bias,
                                           0, 64)
    Q = torch.from_numpy(f64(q)).permute(0, 2, 1, 3)
    K = torch.from_numpy(f64(k)).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    V = torch.from_numpy(f64(v)).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
    np.testing.assert_allclose(out.reshape(B, T, Hq, d), ref.permute(0, 2, 1, 3).numpy(),
                               rtol=0, atol=1e-12)


def test_constant_bias_leaves_output_unchanged(oracle_mod):
    B, T, Hq, Hkv, d = 1, 27, 4, 1, 128
    q, k, v = rand_bf16((B, T, Hq, d)), rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    # dyadic bias so that adding the constant is exact in fp32
    b0 = (np.round(rng.standard_normal((Hq, 33)) * 1024) / 1024).astype(np.float32)
    C = Hkv * d
    w = identity_taps(C)
    base, lse0, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b0, 9, 32)
    shift = np.float32(2.5)
    shifted, lse1, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b0 + shift, 9, 32)
    np.testing.assert_allclose(shifted, base, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse1 - lse0, 2.5, rtol=0, atol=1e-6)


def test_window_equals_minus_infinity_bias(oracle_mod):
    B, T, Hq, Hkv, d, W = 1, 40, 4, 2, 128, 6
    q, k, v = rand_bf16((B, T, Hq, d)), rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    D_max = T
    b = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    bw = b.copy()
    bw[:, W:] = -np.inf
    w = identity_taps(Hkv * d)
    win, _, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, W, D_max)
    inf, _, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, bw, 0, D_max)
    np.testing.assert_allclose(win, inf, rtol=0, atol=1e-13)


def test_zero_query_closed_form(oracle_mod):
    # q = 0: out_i = sum_j softmax_j(bias[h, min(i-j, D_max)]) v_j
    B, T, Hq, Hkv, d, D_max = 1, 45, 4, 2, 128, 12
    q = np.zeros((B, T, Hq, d), np.uint16)
    k, v = rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    b = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    w = identity_taps(Hkv * d)
    out, _, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, 0, D_max)
    out = out.reshape(B, T, Hq, d)
    vf = f64(v)
    for h in range(Hq):
        for i in range(T):
            logits = np.array([b[h, min(i - j, D_max)] for j in range(i + 1)], np.float64)
            p = np.exp(logits - logits.max())
            p /= p.sum()
            ref = p @ vf[0, : i + 1, h // (Hq // Hkv), :]
            np.testing.assert_allclose(out[0, i, h], ref, rtol=0, atol=1e-12)


def test_one_hot_bias_selects_key_at_that_distance(oracle_mod):
    # a +40 bias at distance 3 makes row i copy v[i-3]: pins i-j (not j-i)
    B, T, Hq, Hkv, d, D_max, delta = 1, 20, 2, 1, 128, 16, 3
    q = np.zeros((B, T, Hq, d), np.uint16)
    k, v = rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    b = np.zeros((Hq, D_max + 1), np.float32)
    b[:, delta] = 40.0
    w = identity_taps(d)
    out, _, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, 0, D_max)
    out = out.reshape(B, T, Hq, d)
    vf = f64(v)
    for i in range(delta, T):
        np.testing.assert_allclose(out[0, i, 0], vf[0, i - delta, 0], rtol=0, atol=1e-14)


def test_clip_at_dmax(oracle_mod):
    # every key at distance >= D_max takes the bias entry b[h, D_max]
    B, T, Hq, Hkv, d, D_max = 1, 30, 2, 1, 128, 4
    q = np.zeros((B, T, Hq, d), np.uint16)
    k, v = rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    b = np.zeros((Hq, D_max + 1), np.float32)
    b[:, D_max] = 5.0
    w = identity_taps(d)
    out, lse, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, 0, D_max)
    lse = lse.reshape(T, Hq)
    for i in range(T):
        far = max(0, i - D_max + 1)            # keys at distance >= D_max
        expected = math.log((i + 1 - far) + far * math.exp(5.0))
        assert abs(lse[i, 0] - expected) < 1e-9


def test_gqa_grouping_is_contiguous(oracle_mod):
    # head h reads kv head h // (Hq/Hkv): zero all kv heads but one
    B, T, Hq, Hkv, d = 1, 12, 8, 4, 128
    q = rand_bf16((B, T, Hq, d))
    k = rand_bf16((B, T, Hkv, d))
    v = np.zeros((B, T, Hkv, d), np.uint16)
    v[:, :, 2, :] = bf16_bits(np.ones((B, T, d), np.float32))
    b = np.zeros((Hq, 17), np.float32)
    w = identity_taps(Hkv * d)
    out, _, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, 0, 16)
    out = out.reshape(B, T, Hq, d)
    for h in range(Hq):
        exp = 1.0 if h // 2 == 2 else 0.0
        np.testing.assert_allclose(out[0, :, h, :], exp, rtol=0, atol=1e-14)


def test_worked_example_golden(oracle_mod):
    B, T, Hq, Hkv, d, D_max = 1, 4, 2, 1, 128, 2
    q = np.zeros((B, T, Hq, d), np.uint16)
    k = bf16_bits(np.ones((B, T, Hkv, d), np.float32))
    v = bf16_bits(np.broadcast_to(np.arange(1, T + 1, dtype=np.float32)[None, :, None, None],
                                  (B, T, Hkv, d)).copy())
    wk = np.zeros((d, 4), np.float32)
    wk[:, 0] = 1
    wv = np.zeros((d, 4), np.float32)
    wv[:, 0] = 1
    wv[:, 1] = 1
    bias = np.array([[0.0, math.log(2), math.log(4)], [0.0, 0.0, 0.0]], np.float32)
    results = {}
    for W in (0, 2):
        out, lse, _, vc = oracle_mod.prefill_rows(q, k, v, wk, wv, bias, W, D_max)
        assert np.array_equal(f64(vc[0, :, 0, 0]), [1.0, 3.0, 5.0, 7.0])
        results[W] = (out.reshape(T, Hq, d), lse.reshape(T, Hq))
    n = 0
    with open(os.path.join(GOLDEN, "worked_example.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            W, h, i, frac, explse = line.split()
            W, h, i = int(W), int(h), int(i)
            val = float(Fraction(frac))
            out, lse = results[W]
            np.testing.assert_allclose(out[i, h], val, rtol=1e-6)
            assert abs(lse[i, h] - math.log(float(explse))) < 1e-6
            n += 1
    assert n == 16


def test_brute_force_python_rows(oracle_mod):
    # pure-Python enumeration of the definition on a tiny case, with exp from
    # the math module and sums in a different order (reverse key order)
    B, T, Hq, Hkv, d, W, D_max = 1, 9, 2, 1, 128, 4, 5
    q, k, v = rand_bf16((B, T, Hq, d)), rand_bf16((B, T, Hkv, d)), rand_bf16((B, T, Hkv, d))
    b = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    w = identity_taps(d)
    out, _, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, W, D_max)
    out = out.reshape(T, Hq, d)
    qf, kf, vf = f64(q)[0], f64(k)[0], f64(v)[0]
    for h in range(Hq):
        for i in range(T):
            keys = [j for j in range(T) if 0 <= i - j < W]
            logit = {j: sum(qf[i, h, e] * kf[j, 0, e] for e in range(d)) / math.sqrt(d)
                     + float(b[h, min(i - j, D_max)]) for j in keys}
            z = sum(math.exp(logit[j]) for j in reversed(keys))
            for e in (0, 17, 127):
                ref = sum(math.exp(logit[j]) * vf[j, 0, e] for j in reversed(keys)) / z
                assert abs(out[i, h, e] - ref) < 1e-12


def test_decode_equals_prefill_last_row_and_block_order(oracle_mod):
    # the paged single-token decode at length L equals prefill row L-1, for
    # any placement of the blocks in the pool
    S, Hq, Hkv, d, W, D_max = 2, 4, 2, 128, 100, 200
    T = 260
    q = rand_bf16((S, T, Hq, d))
    k, v = rand_bf16((S, T, Hkv, d)), rand_bf16((S, T, Hkv, d))
    b = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    w = identity_taps(Hkv * d)
    rows = np.array([[s, h, T - 1] for s in range(S) for h in range(Hq)], np.int32)
    ref, ref_lse, _, _ = oracle_mod.prefill_rows(q, k, v, w, w, b, W, D_max, rows)
    nb = 3
    for trial in range(2):
        perm = rng.permutation(S * nb + 5).astype(np.int32)[: S * nb]
        bt = perm.reshape(S, nb)
        kc = rand_bf16((S * nb + 5, Hkv, 128, d))     # unused slots hold noise
        vc = rand_bf16((S * nb + 5, Hkv, 128, d))
        for s in range(S):
            for j in range(T):
                kc[bt[s, j // 128], :, j % 128] = k[s, j]
                vc[bt[s, j // 128], :, j % 128] = v[s, j]
        out, lse = oracle_mod.decode_rows(q[:, T - 1], kc, vc, bt, np.full(S, T, np.int32), b,
                                          W, D_max)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("Q,W,D_max", [(1, 0, 300), (3, 100, 200), (9, 0, 40), (9, 7, 300)])
def test_decode_mq_equals_prefill_rows(oracle_mod, Q, W, D_max):
    # q_len draft tokens appended at the end of a sequence of length T: query
    # qi sits at T - Q + qi, sees keys up to itself (inside the window) and
    # gets the bias at its own distance; this must equal the prefill rows of
    # the same positions, for any placement of the blocks in the pool, with the
    # cache holding the prefill's post-sconv keys and values
    S, Hq, Hkv, d = 2, 4, 2, 128
    T = 261
    C = Hkv * d
    q = rand_bf16((S, T, Hq, d))
    k, v = rand_bf16((S, T, Hkv, d)), rand_bf16((S, T, Hkv, d))
    wk = rng.standard_normal((C, 4)).astype(np.float32) * 0.5
    wv = rng.standard_normal((C, 4)).astype(np.float32) * 0.5
    b = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    rows = np.array([[s, h, i] for s in range(S) for i in range(T - Q, T) for h in range(Hq)],
                    np.int32)
    ref, ref_lse, kc_all, vc_all = oracle_mod.prefill_rows(q, k, v, wk, wv, b, W, D_max)
    ref = ref.reshape(S, T, Hq, d)
    ref_lse = ref_lse.reshape(S, T, Hq)
    kc_all = kc_all.reshape(S, T, Hkv, d)
    vc_all = vc_all.reshape(S, T, Hkv, d)
    nb = 3
    perm = rng.permutation(S * nb + 4).astype(np.int32)[: S * nb]
    bt = perm.reshape(S, nb)
    kc = rand_bf16((S * nb + 4, Hkv, 128, d))     # unused slots hold noise
    vc = rand_bf16((S * nb + 4, Hkv, 128, d))
    for s in range(S):
        for j in range(T):
            kc[bt[s, j // 128], :, j % 128] = kc_all[s, j]
            vc[bt[s, j // 128], :, j % 128] = vc_all[s, j]
    out, lse = oracle_mod.decode_mq_rows(q[:, T - Q:], kc, vc, bt, np.full(S, T, np.int32), b,
                                         W, D_max)
    np.testing.assert_allclose(out.reshape(S, Q, Hq, d), ref[:, T - Q:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(S, Q, Hq), ref_lse[:, T - Q:], rtol=0, atol=1e-12)
    assert rows.shape[0] == S * Q * Hq


def test_decode_mq_single_token_equals_decode(oracle_mod):
    S, Hq, Hkv, d, W, D_max = 3, 8, 2, 128, 50, 64
    nb = 2
    lens = np.array([1, 130, 256], np.int32)
    q = rand_bf16((S, Hq, d))
    kc, vc = rand_bf16((S * nb, Hkv, 128, d)), rand_bf16((S * nb, Hkv, 128, d))
    bt = rng.permutation(S * nb).astype(np.int32).reshape(S, nb)
    b = rng.standard_normal((Hq, D_max + 1)).astype(np.float32)
    one, lse1 = oracle_mod.decode_rows(q, kc, vc, bt, lens, b, W, D_max)
    mq, lse2 = oracle_mod.decode_mq_rows(q[:, None], kc, vc, bt, lens, b, W, D_max)
    np.testing.assert_array_equal(mq, one)
    np.testing.assert_array_equal(lse2, lse1)
