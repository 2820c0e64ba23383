"""fp64 CPU oracle for the Inkling decoder attention layer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg may use this package; the product path (the CUDA library and
its Python binding) never imports it, and this package imports nothing from
the product.  The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over
independent rows); this module only builds it with gcc and marshals numpy
arrays into it.

Sources for what is computed: vLLM Recipes page "thinkingmachines/Inkling",
section Overview (Attention and Short convolution bullets) and the MI355X
launch line in section Client Usage (``--block-size 128``); bitbyai.com
"TML Inkling on vLLM", section "What makes Inkling different?".  bf16 values
cross this interface as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc, -O2, OpenMP).

    -ffp-contract=off keeps every product and sum a separately rounded fp64
    operation, as written in the source."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-std=c11", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int64
            lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_f64.restype = ctypes.c_double
            lib.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
            lib.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
            lib.oracle_num_threads.restype = ctypes.c_int
            lib.oracle_sconv.argtypes = [P, P, P, I, I, I, P]
            lib.oracle_sconv_append.argtypes = [P, P, P, P, P, P, I, I, I, I, I]
            lib.oracle_attention_rows.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, I, P, P]
            lib.oracle_prefill_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P, I,
                                                P, P, P, P]
            lib.oracle_decode_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, P]
            lib.oracle_decode_mq_rows.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P, I, P, P]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"bf16 arrays cross the oracle as uint16 bit patterns, got {a.dtype}")
    return a


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def num_threads() -> int:
    """OpenMP threads the oracle runs on (OMP_NUM_THREADS or all host cores)."""
    return int(_load().oracle_num_threads())


def bf16_to_f64(bits: int) -> float:
    return float(_load().oracle_bf16_to_f64(int(bits)))


def f64_to_bf16(x: float) -> int:
    """One rounding, to nearest with ties to even."""
    return int(_load().oracle_f64_to_bf16_rne(float(x)))


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (pure bit manipulation)."""
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sconv(x: np.ndarray, w: np.ndarray, hist: np.ndarray | None = None) -> np.ndarray:
    """Causal depthwise window-4 short convolution.

    x [B, T, C] bf16 bits; w [C, 4] fp32 (tap 0 = current token);
    hist [B, 3, C] bf16 bits (oldest first) or None for zero history.
    Returns y [B, T, C] bf16 bits."""
    x = _u16(x)
    B, T, C = x.shape
    w = _f32(w).reshape(C, 4)
    h = None if hist is None else _u16(hist).reshape(B, 3, C)
    y = np.empty_like(x)
    _load().oracle_sconv(_ptr(x), _ptr(h), _ptr(w), B, T, C, _ptr(y))
    return y


def sconv_append(x_new, state, w, cache, block_table, seq_lens):
    """Decode-side append (in place on ``state`` and ``cache``).

    x_new [S, n_new, Hkv, d] bf16 bits; state [S, 3, Hkv*d] bf16 bits;
    w [Hkv*d, 4] fp32; cache [num_blocks, Hkv, 128, d] bf16 bits;
    block_table [S, max_blocks] int32; seq_lens [S] int32 (after append)."""
    x_new = _u16(x_new)
    S, n_new, Hkv, d = x_new.shape
    if not (state.flags["C_CONTIGUOUS"] and cache.flags["C_CONTIGUOUS"]):
        raise ValueError("state and cache are updated in place and must be contiguous")
    if state.dtype != np.uint16 or cache.dtype != np.uint16:
        raise TypeError("state and cache are bf16 bit patterns (uint16)")
    bt = _i32(block_table)
    sl = _i32(seq_lens)
    _load().oracle_sconv_append(_ptr(x_new), _ptr(state), _ptr(_f32(w)), _ptr(cache),
                                _ptr(bt), _ptr(sl), S, n_new, Hkv, d, bt.shape[1])


def attention_rows(q, kc, vc, bias, window, D_max, rows):
    """Attention over post-sconv keys/values for the listed (b, h, i) rows.

    q [B, T, Hq, d], kc/vc [B, T, Hkv, d] bf16 bits; bias [Hq, D_max+1] fp32;
    rows int array [n, 3].  Returns (out [n, d] fp64, lse [n] fp64)."""
    q, kc, vc = _u16(q), _u16(kc), _u16(vc)
    B, T, Hq, d = q.shape
    Hkv = kc.shape[2]
    bias = _f32(bias)
    assert bias.shape == (Hq, D_max + 1)
    rows = _i32(rows).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    _load().oracle_attention_rows(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bias), B, T, Hq, Hkv,
                                  d, int(window), int(D_max), _ptr(rows), n, _ptr(out),
                                  _ptr(lse))
    return out, lse


def prefill_rows(q, k_raw, v_raw, w_k, w_v, bias, window, D_max, rows=None):
    """Prefill: zero-history sconv of raw keys/values, then attention rows.

    rows None means every (b, i, h) row in [B, T, Hq] order.  Returns
    (out [n, d] fp64, lse [n] fp64, kc, vc) with kc/vc the bf16 post-sconv
    keys/values [B, T, Hkv, d]."""
    q, k_raw, v_raw = _u16(q), _u16(k_raw), _u16(v_raw)
    B, T, Hq, d = q.shape
    Hkv = k_raw.shape[2]
    bias = _f32(bias)
    assert bias.shape == (Hq, D_max + 1)
    if rows is None:
        bb, ii, hh = np.meshgrid(np.arange(B), np.arange(T), np.arange(Hq), indexing="ij")
        rows = np.stack([bb.ravel(), hh.ravel(), ii.ravel()], axis=1)
    rows = _i32(rows).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    kc = np.empty_like(k_raw)
    vc = np.empty_like(v_raw)
    _load().oracle_prefill_rows(_ptr(q), _ptr(k_raw), _ptr(v_raw), _ptr(_f32(w_k)),
                                _ptr(_f32(w_v)), _ptr(bias), B, T, Hq, Hkv, d, int(window),
                                int(D_max), _ptr(rows), n, _ptr(out), _ptr(lse), _ptr(kc),
                                _ptr(vc))
    return out, lse, kc, vc


def decode_rows(q, k_cache, v_cache, block_table, seq_lens, bias, window, D_max, pairs=None):
    """Single-token decode at position L-1 through the paged cache.

    q [S, Hq, d] bf16 bits; caches [num_blocks, Hkv, 128, d] bf16 bits;
    pairs int array [n, 2] of (s, h), None for all in [S, Hq] order.
    Returns (out [n, d] fp64, lse [n] fp64)."""
    q, k_cache, v_cache = _u16(q), _u16(k_cache), _u16(v_cache)
    S, Hq, d = q.shape
    Hkv = k_cache.shape[1]
    assert k_cache.shape[2] == 128
    bt = _i32(block_table)
    sl = _i32(seq_lens)
    bias = _f32(bias)
    assert bias.shape == (Hq, D_max + 1)
    if pairs is None:
        ss, hh = np.meshgrid(np.arange(S), np.arange(Hq), indexing="ij")
        pairs = np.stack([ss.ravel(), hh.ravel()], axis=1)
    pairs = _i32(pairs).reshape(-1, 2)
    n = pairs.shape[0]
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    _load().oracle_decode_rows(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt), _ptr(sl),
                               _ptr(bias), Hq, Hkv, d, bt.shape[1], int(window), int(D_max),
                               _ptr(pairs), n, _ptr(out), _ptr(lse))
    return out, lse


def decode_mq_rows(q, k_cache, v_cache, block_table, seq_lens, bias, window, D_max, rows=None):
    """Multi-token decode: query qi of sequence s sits at position L_s - q_len + qi.

    q [S, q_len, Hq, d] bf16 bits; caches [num_blocks, Hkv, 128, d] bf16 bits;
    rows int array [n, 3] of (s, qi, h), None for all in [S, q_len, Hq] order.
    Returns (out [n, d] fp64, lse [n] fp64)."""
    q, k_cache, v_cache = _u16(q), _u16(k_cache), _u16(v_cache)
    S, Q, Hq, d = q.shape
    Hkv = k_cache.shape[1]
    assert k_cache.shape[2] == 128
    bt = _i32(block_table)
    sl = _i32(seq_lens)
    assert (sl >= Q).all(), "every sequence holds its q_len new tokens"
    bias = _f32(bias)
    assert bias.shape == (Hq, D_max + 1)
    if rows is None:
        ss, qq, hh = np.meshgrid(np.arange(S), np.arange(Q), np.arange(Hq), indexing="ij")
        rows = np.stack([ss.ravel(), qq.ravel(), hh.ravel()], axis=1)
    rows = _i32(rows).reshape(-1, 3)
    n = rows.shape[0]
    out = np.empty((n, d), np.float64)
    lse = np.empty((n,), np.float64)
    _load().oracle_decode_mq_rows(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt), _ptr(sl),
                                  _ptr(bias), Hq, Hkv, d, bt.shape[1], int(window), int(D_max),
                                  Q, _ptr(rows), n, _ptr(out), _ptr(lse))
    return out, lse
