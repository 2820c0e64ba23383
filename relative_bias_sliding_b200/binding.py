"""Python binding of libinkling (ctypes): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module checks
torch tensors (device, dtype, shape, contiguity), turns them into pointers and
sizes, and calls the C ABI declared in include/inkling.h on the current torch
stream.  It never computes a result itself and has no CPU fallback: if the
library is missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libinkling.so")

INKLING_OK, INKLING_ERR_INVALID, INKLING_ERR_UNSUPPORTED, INKLING_ERR_CUDA = 0, 1, 2, 3
STATUS_TIMEOUT, STATUS_BAD_BLOCK, STATUS_BAD_LENGTH = 1, 2, 4
HEAD_DIM = 128
BLOCK_SIZE = 128
INKLING_PREFILL_TWO_PASS_MIN_TOKENS = 2048
INKLING_PREFILL_TWO_PASS_MIN_T = 512

EXPORTED = (
    "inkling_last_error",
    "inkling_version",
    "inkling_selftest_wait_timeout",
    "inkling_sconv_kv",
    "inkling_sconv_out",
    "inkling_sconv_out_sharded",
    "inkling_attn_prefill",
    "inkling_attn_prefill_paged",
    "inkling_attn_prefill_workspace_bytes",
    "inkling_attn_decode_workspace_bytes",
    "inkling_attn_decode_num_splits",
    "inkling_attn_decode",
    "inkling_attn_decode_static",
)

_P = ctypes.c_void_p
_I = ctypes.c_int32


class SconvParams(ctypes.Structure):
    _fields_ = [("k_new", _P), ("v_new", _P), ("w_k", _P), ("w_v", _P), ("k_state", _P),
                ("v_state", _P), ("k_cache", _P), ("v_cache", _P), ("block_table", _P),
                ("seq_lens", _P), ("status", _P), ("num_seqs", _I), ("n_new", _I),
                ("num_kv_heads", _I), ("head_dim", _I), ("max_blocks", _I), ("num_blocks", _I)]


class PrefillParams(ctypes.Structure):
    _fields_ = [("q", _P), ("k_raw", _P), ("v_raw", _P), ("w_k", _P), ("w_v", _P), ("bias", _P),
                ("out", _P), ("lse", _P), ("status", _P), ("batch", _I), ("seq_len", _I),
                ("num_q_heads", _I), ("num_kv_heads", _I), ("head_dim", _I), ("window", _I),
                ("d_max", _I), ("k_cache", _P), ("v_cache", _P), ("block_table", _P),
                ("max_blocks", _I), ("num_blocks", _I), ("k_state", _P), ("v_state", _P),
                ("path", _I), ("workspace", _P), ("workspace_bytes", ctypes.c_size_t)]


# inkling_attn_prefill execution paths (INKLING_PREFILL_*)
PREFILL_PATHS = {"auto": 0, "fused": 1, "two_pass": 2}


class SconvOutParams(ctypes.Structure):
    _fields_ = [("x", _P), ("w", _P), ("state", _P), ("y", _P), ("batch", _I), ("seq_len", _I),
                ("channels", _I)]


SHARD_MAX_RANKS = 8


class SconvOutShardedParams(ctypes.Structure):
    _fields_ = [("x_parts", ctypes.POINTER(_P)), ("y_parts", ctypes.POINTER(_P)), ("w", _P),
                ("state", _P), ("n_ranks", _I), ("rank", _I), ("batch", _I), ("seq_len", _I),
                ("channels", _I)]


class PrefillPagedParams(ctypes.Structure):
    _fields_ = [("q", _P), ("cu_q", _P), ("k_cache", _P), ("v_cache", _P), ("block_table", _P),
                ("seq_lens", _P), ("bias", _P), ("out", _P), ("lse", _P), ("status", _P),
                ("num_seqs", _I), ("total_q", _I), ("max_q", _I), ("num_q_heads", _I),
                ("num_kv_heads", _I), ("head_dim", _I), ("max_blocks", _I), ("num_blocks", _I),
                ("window", _I), ("d_max", _I)]


class DecodeParams(ctypes.Structure):
    _fields_ = [("q", _P), ("k_cache", _P), ("v_cache", _P), ("block_table", _P),
                ("seq_lens", _P), ("bias", _P), ("out", _P), ("lse", _P), ("status", _P),
                ("num_seqs", _I), ("num_q_heads", _I), ("num_kv_heads", _I), ("head_dim", _I),
                ("max_blocks", _I), ("num_blocks", _I), ("window", _I), ("d_max", _I),
                ("num_splits", _I), ("q_len", _I)]


class InklingError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libinkling error {code}: {msg}")
        self.code = code


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load libinkling.so and declare its signatures (raises if it is absent)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is not built: run `python -m relative_bias_sliding_b200.build`")
        lib = ctypes.CDLL(path)
        lib.inkling_last_error.restype = ctypes.c_char_p
        lib.inkling_version.restype = ctypes.c_int
        lib.inkling_selftest_wait_timeout.argtypes = [_P, ctypes.c_uint32, _P]
        lib.inkling_selftest_wait_timeout.restype = ctypes.c_int
        lib.inkling_sconv_kv.argtypes = [ctypes.POINTER(SconvParams), _P]
        lib.inkling_sconv_kv.restype = ctypes.c_int
        lib.inkling_attn_prefill.argtypes = [ctypes.POINTER(PrefillParams), _P]
        lib.inkling_attn_prefill.restype = ctypes.c_int
        lib.inkling_attn_prefill_workspace_bytes.argtypes = [ctypes.POINTER(PrefillParams)]
        lib.inkling_attn_prefill_workspace_bytes.restype = ctypes.c_size_t
        lib.inkling_sconv_out.argtypes = [ctypes.POINTER(SconvOutParams), _P]
        lib.inkling_sconv_out.restype = ctypes.c_int
        lib.inkling_sconv_out_sharded.argtypes = [ctypes.POINTER(SconvOutShardedParams), _P]
        lib.inkling_sconv_out_sharded.restype = ctypes.c_int
        lib.inkling_attn_prefill_paged.argtypes = [ctypes.POINTER(PrefillPagedParams), _P]
        lib.inkling_attn_prefill_paged.restype = ctypes.c_int
        lib.inkling_attn_decode_workspace_bytes.argtypes = [_I, _I, _I]
        lib.inkling_attn_decode_workspace_bytes.restype = ctypes.c_size_t
        lib.inkling_attn_decode_num_splits.argtypes = [ctypes.POINTER(DecodeParams)]
        lib.inkling_attn_decode_num_splits.restype = _I
        lib.inkling_attn_decode.argtypes = [ctypes.POINTER(DecodeParams), _P, ctypes.c_size_t, _P]
        lib.inkling_attn_decode.restype = ctypes.c_int
        lib.inkling_attn_decode_static.argtypes = [ctypes.POINTER(DecodeParams), _P]
        lib.inkling_attn_decode_static.restype = ctypes.c_int
        _lib = lib
        return lib


def _check(code):
    if code != INKLING_OK:
        raise InklingError(code, load_library().inkling_last_error().decode())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, dtype, name, ndim=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def sconv_kv(k_new, v_new, w_k, w_v, k_state, v_state, k_cache, v_cache, block_table, seq_lens,
             status=None, stream=None):
    """Decode-side sconv append (in place on the states and caches)."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    _dev(k_new, bf, "k_new", 4), _dev(v_new, bf, "v_new", 4)
    S, n_new, Hkv, d = k_new.shape
    if v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new shapes differ")
    for n, t in (("w_k", w_k), ("w_v", w_v)):
        _dev(t, f32, n)
        if t.shape != (Hkv * d, 4):
            raise ValueError(f"{n} must be [{Hkv * d}, 4]")
    for n, t in (("k_state", k_state), ("v_state", v_state)):
        _dev(t, bf, n)
        if t.shape != (S, 3, Hkv * d):
            raise ValueError(f"{n} must be [{S}, 3, {Hkv * d}]")
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        _dev(t, bf, n, 4)
        if t.shape[1:] != (Hkv, BLOCK_SIZE, d):
            raise ValueError(f"{n} must be [num_blocks, {Hkv}, 128, {d}]")
    _dev(block_table, i32, "block_table", 2), _dev(seq_lens, i32, "seq_lens", 1)
    _dev(status, i32, "status")
    p = SconvParams(_ptr(k_new), _ptr(v_new), _ptr(w_k), _ptr(w_v), _ptr(k_state), _ptr(v_state),
                    _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens), _ptr(status),
                    S, n_new, Hkv, d, block_table.shape[1], k_cache.shape[0])
    _check(load_library().inkling_sconv_kv(ctypes.byref(p), _stream(stream)))


def attn_prefill(q, k_raw, v_raw, w_k, w_v, bias, window=0, out=None, lse=None, status=None,
                 stream=None, k_cache=None, v_cache=None, block_table=None, k_state=None,
                 v_state=None, path="auto", workspace=None):
    """Prefill attention over whole prompts, the sconv of the raw keys/values
    included; returns ``out`` [B, T, Hq, d] bf16.

    With ``k_cache``, ``v_cache`` [num_blocks, Hkv, 128, d] and ``block_table``
    [B, max_blocks] the call also writes the post-sconv keys/values of tokens
    0..T-1 into the paged cache; with ``k_state``, ``v_state`` [B, 3, Hkv*d]
    it writes the new sconv state.

    ``path``: "fused" (one kernel, the sconv applied to each tile on its way
    to the tensor cores), "two_pass" (the sconv written once in the paged
    layout, then the paged prefill kernel) or "auto" (the library's choice by
    length).  Without a cache the two-pass path needs scratch: ``workspace``
    (a uint8 CUDA tensor of at least ``prefill_workspace_bytes`` bytes), or
    one is allocated here."""
    bf, f32 = torch.bfloat16, torch.float32
    _dev(q, bf, "q", 4), _dev(k_raw, bf, "k_raw", 4), _dev(v_raw, bf, "v_raw", 4)
    B, T, Hq, d = q.shape
    Hkv = k_raw.shape[2]
    if k_raw.shape != (B, T, Hkv, d) or v_raw.shape != k_raw.shape:
        raise ValueError("k_raw / v_raw must be [B, T, Hkv, d] matching q")
    for n, t in (("w_k", w_k), ("w_v", w_v)):
        _dev(t, f32, n)
        if t.shape != (Hkv * d, 4):
            raise ValueError(f"{n} must be [{Hkv * d}, 4]")
    _dev(bias, f32, "bias", 2)
    if bias.shape[0] != Hq:
        raise ValueError("bias must be [Hq, d_max+1]")
    d_max = bias.shape[1] - 1
    if out is None:
        out = torch.empty_like(q)
    _dev(out, bf, "out", 4)
    if out.shape != q.shape:
        raise ValueError("out must match q")
    if lse is not None:
        _dev(lse, f32, "lse", 3)
        if lse.shape != (B, Hq, T):
            raise ValueError("lse must be [B, Hq, T]")
    _dev(status, torch.int32, "status")
    max_blocks = num_blocks = 0
    if k_cache is not None or v_cache is not None or block_table is not None:
        if k_cache is None or v_cache is None or block_table is None:
            raise ValueError("k_cache, v_cache and block_table go together")
        for n, t in (("k_cache", k_cache), ("v_cache", v_cache)):
            _dev(t, bf, n, 4)
            if t.shape[1:] != (Hkv, BLOCK_SIZE, d):
                raise ValueError(f"{n} must be [num_blocks, {Hkv}, {BLOCK_SIZE}, {d}]")
        _dev(block_table, torch.int32, "block_table", 2)
        if block_table.shape[0] != B:
            raise ValueError("block_table must be [B, max_blocks]")
        max_blocks, num_blocks = block_table.shape[1], k_cache.shape[0]
    for n, t in (("k_state", k_state), ("v_state", v_state)):
        if t is not None:
            _dev(t, bf, n, 3)
            if t.shape != (B, 3, Hkv * d):
                raise ValueError(f"{n} must be [{B}, 3, {Hkv * d}]")
    if path not in PREFILL_PATHS:
        raise ValueError(f"path must be one of {sorted(PREFILL_PATHS)}")
    p = PrefillParams(_ptr(q), _ptr(k_raw), _ptr(v_raw), _ptr(w_k), _ptr(w_v), _ptr(bias),
                      _ptr(out), _ptr(lse), _ptr(status), B, T, Hq, Hkv, d, int(window), d_max,
                      _ptr(k_cache), _ptr(v_cache), _ptr(block_table), max_blocks, num_blocks,
                      _ptr(k_state), _ptr(v_state), PREFILL_PATHS[path], None, 0)
    lib = load_library()
    need = lib.inkling_attn_prefill_workspace_bytes(ctypes.byref(p))
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        _dev(workspace, torch.uint8, "workspace", 1)
        p.workspace, p.workspace_bytes = _ptr(workspace), workspace.numel()
    _check(lib.inkling_attn_prefill(ctypes.byref(p), _stream(stream)))
    return out


def prefill_workspace_bytes(batch, seq_len, num_q_heads, num_kv_heads, path="auto",
                            with_cache=False):
    """Bytes of scratch ``attn_prefill`` uses for these sizes and path (0 when
    it needs none: the fused path, or a cache given)."""
    if path not in PREFILL_PATHS:
        raise ValueError(f"path must be one of {sorted(PREFILL_PATHS)}")
    p = PrefillParams()
    p.batch, p.seq_len, p.num_q_heads, p.num_kv_heads = batch, seq_len, num_q_heads, num_kv_heads
    p.head_dim, p.path = 128, PREFILL_PATHS[path]
    p.k_cache = 16 if with_cache else None  # only tested against NULL
    return int(load_library().inkling_attn_prefill_workspace_bytes(ctypes.byref(p)))


def sconv_out(x, w, state=None, out=None, stream=None):
    """Output sconv: x [B, T, C] bf16 (attention output, C = Hq*128), taps w
    [C, 4] fp32; state [B, 3, C] bf16 (updated in place) or None for zero
    history.  Returns y [B, T, C] bf16."""
    _dev(x, torch.bfloat16, "x", 3)
    B, T, C = x.shape
    _dev(w, torch.float32, "w", 2)
    if w.shape != (C, 4):
        raise ValueError(f"w must be [{C}, 4]")
    if state is not None:
        _dev(state, torch.bfloat16, "state", 3)
        if state.shape != (B, 3, C):
            raise ValueError(f"state must be [{B}, 3, {C}]")
    if out is None:
        out = torch.empty_like(x)
    _dev(out, torch.bfloat16, "out", 3)
    if out.shape != x.shape:
        raise ValueError("out must match x")
    p = SconvOutParams(_ptr(x), _ptr(w), _ptr(state), _ptr(out), B, T, C)
    _check(load_library().inkling_sconv_out(ctypes.byref(p), _stream(stream)))
    return out


def sconv_out_sharded(x_parts, w, y_parts, rank, state=None, stream=None):
    """One rank's call of the output sconv sharded over channels, fused with
    its reduce-scatter and all-gather (see inkling.h).  ``x_parts`` /
    ``y_parts``: one [B, T, C] bf16 tensor per rank (the partial sums and the
    outputs), each readable / writable from this device; ``state``: this
    rank's [B, 3, C / n] shard of the sconv state or None.  Writes channels
    [rank * C/n, (rank+1) * C/n) of the sconv of the summed input into every
    y_parts[r]; the caller orders the ranks' calls (inputs complete before,
    outputs read after every rank's call)."""
    n = len(x_parts)
    if n < 1 or n > SHARD_MAX_RANKS or len(y_parts) != n:
        raise ValueError(f"x_parts and y_parts must hold the same 1..{SHARD_MAX_RANKS} tensors")
    B, T, C = x_parts[0].shape
    for i, t in enumerate(list(x_parts) + list(y_parts)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or tuple(t.shape) != (B, T, C):
            raise ValueError(f"part {i} must be a bf16 [B, T, C] tensor like x_parts[0]")
        if not t.is_contiguous():
            raise ValueError(f"part {i} must be contiguous")
    _dev(w, torch.float32, "w", 2)
    if w.shape != (C, 4):
        raise ValueError("w must be [C, 4]")
    if state is not None:
        _dev(state, torch.bfloat16, "state", 3)
        if tuple(state.shape) != (B, 3, C // n):
            raise ValueError("state must be [B, 3, C / n_ranks]")
    xs = (_P * n)(*[t.data_ptr() for t in x_parts])
    ys = (_P * n)(*[t.data_ptr() for t in y_parts])
    p = SconvOutShardedParams(xs, ys, _ptr(w), _ptr(state), n, int(rank), B, T, C)
    _check(load_library().inkling_sconv_out_sharded(ctypes.byref(p), _stream(stream)))


def attn_prefill_paged(q, cu_q, k_cache, v_cache, block_table, seq_lens, bias, window=0,
                       max_q=None, out=None, lse=None, status=None, stream=None):
    """Chunked prefill over the paged cache (see inkling.h): ``q`` [total_q, Hq, d]
    packs the new tokens of every sequence (rows cu_q[s] .. cu_q[s+1]-1), whose
    keys and values sconv_kv has already appended; ``seq_lens`` are the lengths
    including them.  ``max_q`` bounds every chunk length (read from ``cu_q``
    with a device sync when not given).  Returns ``out`` [total_q, Hq, d]."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    _dev(q, bf, "q", 3)
    total_q, Hq, d = q.shape
    _dev(cu_q, i32, "cu_q", 1)
    S = cu_q.shape[0] - 1
    if S < 0:
        raise ValueError("cu_q must have num_seqs + 1 entries")
    _dev(k_cache, bf, "k_cache", 4), _dev(v_cache, bf, "v_cache", 4)
    if k_cache.shape != v_cache.shape or k_cache.shape[2] != BLOCK_SIZE or k_cache.shape[3] != d:
        raise ValueError("caches must be [num_blocks, Hkv, 128, d] and equal")
    Hkv = k_cache.shape[1]
    _dev(block_table, i32, "block_table", 2), _dev(seq_lens, i32, "seq_lens", 1)
    if block_table.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_table / seq_lens must have num_seqs rows")
    _dev(bias, f32, "bias", 2)
    if bias.shape[0] != Hq:
        raise ValueError("bias must be [Hq, d_max+1]")
    if out is None:
        out = torch.empty_like(q)
    _dev(out, bf, "out", 3)
    if out.shape != q.shape:
        raise ValueError("out must match q")
    if lse is not None:
        _dev(lse, f32, "lse", 2)
        if lse.shape != (total_q, Hq):
            raise ValueError("lse must be [total_q, Hq]")
    _dev(status, i32, "status")
    if max_q is None:
        max_q = int((cu_q[1:] - cu_q[:-1]).max().item()) if S > 0 else 0
    p = PrefillPagedParams(_ptr(q), _ptr(cu_q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                           _ptr(seq_lens), _ptr(bias), _ptr(out), _ptr(lse), _ptr(status), S,
                           total_q, int(max_q), Hq, Hkv, d, block_table.shape[1],
                           k_cache.shape[0], int(window), bias.shape[1] - 1)
    _check(load_library().inkling_attn_prefill_paged(ctypes.byref(p), _stream(stream)))
    return out


def _decode_params(q, k_cache, v_cache, block_table, seq_lens, bias, window, out, lse, status,
                   num_splits):
    """q [S, Hq, d] (one token per sequence) or [S, q_len, Hq, d] (the q_len
    newest tokens of each sequence, multi-token decode)."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    if not isinstance(q, torch.Tensor) or q.dim() not in (3, 4):
        raise ValueError("q must be [S, Hq, d] or [S, q_len, Hq, d]")
    _dev(q, bf, "q", q.dim())
    if q.dim() == 3:
        S, Hq, d = q.shape
        Q = 1
    else:
        S, Q, Hq, d = q.shape
    _dev(k_cache, bf, "k_cache", 4), _dev(v_cache, bf, "v_cache", 4)
    if k_cache.shape != v_cache.shape or k_cache.shape[2] != BLOCK_SIZE or k_cache.shape[3] != d:
        raise ValueError("caches must be [num_blocks, Hkv, 128, d] and equal")
    Hkv = k_cache.shape[1]
    _dev(block_table, i32, "block_table", 2), _dev(seq_lens, i32, "seq_lens", 1)
    if block_table.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_table / seq_lens must have num_seqs rows")
    _dev(bias, f32, "bias", 2)
    if bias.shape[0] != Hq:
        raise ValueError("bias must be [Hq, d_max+1]")
    _dev(out, bf, "out", q.dim())
    if out.shape != q.shape:
        raise ValueError("out must match q")
    if lse is not None:
        _dev(lse, f32, "lse", q.dim() - 1)
        if lse.shape != q.shape[:-1]:
            raise ValueError("lse must be q.shape[:-1]")
    _dev(status, i32, "status")
    return DecodeParams(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                        _ptr(bias), _ptr(out), _ptr(lse), _ptr(status), S, Hq, Hkv, d,
                        block_table.shape[1], k_cache.shape[0], int(window), bias.shape[1] - 1,
                        int(num_splits), Q if q.dim() == 4 else 0)


def decode_num_splits(q, k_cache, v_cache, block_table, seq_lens, bias, window=0, num_splits=0):
    """Split count the decode call will use (resolves num_splits=0)."""
    out = torch.empty_like(q)
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, bias, window, out, None, None,
                       num_splits)
    n = load_library().inkling_attn_decode_num_splits(ctypes.byref(p))
    if n <= 0:
        raise InklingError(INKLING_ERR_INVALID, load_library().inkling_last_error().decode())
    return int(n)


def decode_workspace_bytes(num_seqs, num_q_heads, num_splits):
    return int(load_library().inkling_attn_decode_workspace_bytes(num_seqs, num_q_heads,
                                                                   num_splits))


def attn_decode(q, k_cache, v_cache, block_table, seq_lens, bias, window=0, out=None, lse=None,
                workspace=None, num_splits=0, status=None, stream=None):
    """Paged decode; returns ``out`` shaped like ``q``: [S, Hq, d] for one token
    per sequence, [S, q_len, Hq, d] for multi-token decode (the q_len newest
    tokens of each sequence, causal among themselves).  ``workspace`` (uint8
    CUDA tensor) is allocated here by torch when not given."""
    if out is None:
        out = torch.empty_like(q)
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, bias, window, out, lse, status,
                       num_splits)
    lib = load_library()
    splits = lib.inkling_attn_decode_num_splits(ctypes.byref(p))
    if splits <= 0:
        _check(INKLING_ERR_INVALID if not lib.inkling_last_error() else INKLING_ERR_INVALID)
    need = lib.inkling_attn_decode_workspace_bytes(p.num_seqs * max(p.q_len, 1), p.num_q_heads,
                                                   splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _dev(workspace, torch.uint8, "workspace")
    _check(lib.inkling_attn_decode(ctypes.byref(p), _ptr(workspace), workspace.numel(),
                                   _stream(stream)))
    return out


def attn_decode_static(q, k_cache, v_cache, block_table, seq_lens, bias, window=0, out=None,
                       lse=None, num_splits=0, status=None, stream=None):
    """Paged decode (one or q_len tokens per sequence, as attn_decode) that uses
    the library's own 8 MiB scratch for the split partials instead of a
    workspace (for callers that cannot allocate).  Calls must not overlap on
    the GPU; returns ``out``."""
    if out is None:
        out = torch.empty_like(q)
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, bias, window, out, lse, status,
                       num_splits)
    _check(load_library().inkling_attn_decode_static(ctypes.byref(p), _stream(stream)))
    return out


def selftest_wait_timeout(status, limit_us=50000, stream=None):
    """Launch a block whose bounded wait must run out (see inkling.h)."""
    _dev(status, torch.int32, "status")
    _check(load_library().inkling_selftest_wait_timeout(_ptr(status), int(limit_us), _stream(stream)))
