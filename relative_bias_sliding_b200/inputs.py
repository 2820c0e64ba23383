"""Seeded synthetic inputs for the Inkling attention layer.

This module holds no arithmetic of the method: it only draws random tensors
with fixed seeds, shapes and distributions, in a fixed order, so that the CUDA
path and the CPU oracle are fed the same arrays.  Distributions follow the
workloads the layer is measured on: bf16 queries/keys/values N(0, 1), sconv
taps fp32 N(0, 0.5) (0.5 is the standard deviation), bias tables fp32
N(0, sigma), paged caches of 128-token blocks placed by a random permutation
of the block pool.

Draw order (one ``torch.Generator`` per workload, seeded with its seed):
prefill  q, k_raw, v_raw, w_k, w_v, bias
decode   q, k_new, v_new, w_k, w_v, bias, k_state, v_state, seq_lens,
         block permutation, k_cache, v_cache
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch

BLOCK = 128  # tokens per paged-KV block


@dataclass(frozen=True)
class PrefillSpec:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    window: int      # 0 = full causal
    D_max: int
    bias_std: float
    seed: int

    @property
    def allowed_pairs(self) -> int:
        """(i, j) pairs inside the causal band / window, per (batch, head)."""
        T, W = self.T, self.window
        if W <= 0 or W >= T:
            return T * (T + 1) // 2
        return W * (W + 1) // 2 + (T - W) * W

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs: 2 contractions of length d per allowed pair."""
        return 4 * self.d * self.Hq * self.B * self.allowed_pairs


@dataclass(frozen=True)
class DecodeSpec:
    name: str
    S: int
    L_min: int
    L_max: int       # lengths drawn uniformly in [L_min, L_max]; equal = fixed
    Hq: int
    Hkv: int
    d: int
    window: int
    D_max: int
    bias_std: float
    seed: int
    n_new: int = 1


@dataclass(frozen=True)
class ChunkSpec:
    """Chunked prefill: B sequences that already hold `prefix` tokens (their
    post-sconv keys/values in the paged cache, their raw last 3 in the sconv
    state) receive `chunk` new tokens each, all of them queries."""
    name: str
    B: int
    prefix: int
    chunk: int
    Hq: int
    Hkv: int
    d: int
    window: int
    D_max: int
    bias_std: float
    seed: int

    @property
    def allowed_pairs(self) -> int:
        """(query, key) pairs of the chunk rows inside the band / window, per (seq, head)."""
        W, tot = self.window, 0
        for i in range(self.prefix, self.prefix + self.chunk):
            tot += min(i + 1, W) if W > 0 else i + 1
        return tot

    @property
    def flops(self) -> int:
        return 4 * self.d * self.Hq * self.B * self.allowed_pairs


@dataclass(frozen=True)
class SconvOutSpec:
    """Output sconv over the attention output [B, T, Hq*128] with a state."""
    name: str
    B: int
    T: int
    C: int
    seed: int

    @property
    def bytes_moved(self) -> int:
        """x read once and y written once (bf16); the state is negligible."""
        return 2 * self.B * self.T * self.C * 2


WORKLOADS = {
    # tiny full-causal prefill, small enough for the oracle on every row
    "prefill_tiny_b1_t256": PrefillSpec("prefill_tiny_b1_t256", 1, 256, 8, 1, 128, 0, 256,
                                        1.0, 0),
    # sliding-window prefill, window 4096
    "prefill_swa_b4_t8192": PrefillSpec("prefill_swa_b4_t8192", 4, 8192, 64, 8, 128, 4096,
                                        4096, 1.0, 1),
    # full-attention prefill, 32k tokens
    "prefill_full_b1_t32768": PrefillSpec("prefill_full_b1_t32768", 1, 32768, 64, 8, 128, 0,
                                          32768, 0.5, 2),
    # sliding-window decode over 64 sequences of mixed length
    "decode_swa_s64": DecodeSpec("decode_swa_s64", 64, 1024, 32768, 64, 8, 128, 4096, 4096,
                                 1.0, 3),
    # 1M-token full-attention decode, batch 1 and batch 8
    "decode_full_1m_b1": DecodeSpec("decode_full_1m_b1", 1, 1 << 20, 1 << 20, 64, 8, 128, 0,
                                    1 << 20, 0.5, 4),
    "decode_full_1m_b8": DecodeSpec("decode_full_1m_b8", 8, 1 << 20, 1 << 20, 64, 8, 128, 0,
                                    1 << 20, 0.5, 4),
    # sliding-window decode verifying 9 draft tokens per sequence (multi-token
    # prediction: up to 9 tokens per forward step)
    "decode_mtp9_swa_s64": DecodeSpec("decode_mtp9_swa_s64", 64, 1024, 32768, 64, 8, 128, 4096,
                                      4096, 1.0, 3, n_new=9),
    # chunked prefill: 4 sequences with a 6144-token prefix take their last
    # 2048-token chunk (the sliding-window prefill's shape, cut in chunks)
    "prefill_chunked_swa_b4_c2048": ChunkSpec("prefill_chunked_swa_b4_c2048", 4, 6144, 2048, 64,
                                              8, 128, 4096, 4096, 1.0, 5),
    # the sliding-window prefill's shape (B4, T8192, window 4096) taken as one
    # chunk over an empty cache: sconv append into the paged cache, then the
    # paged prefill (zero sconv history)
    "prefill_paged_swa_b4_t8192": ChunkSpec("prefill_paged_swa_b4_t8192", 4, 0, 8192, 64, 8,
                                            128, 4096, 4096, 1.0, 1),
    # output sconv over the sliding-window prefill's attention output
    "sconv_out_b4_t8192": SconvOutSpec("sconv_out_b4_t8192", 4, 8192, 64 * 128, 6),
    # smaller cuts of the same workloads for profiler captures (still larger
    # than L2, a few GB on the device at most)
    "prefill_swa_b1_t8192": PrefillSpec("prefill_swa_b1_t8192", 1, 8192, 64, 8, 128, 4096,
                                        4096, 1.0, 1),
    "decode_swa_s16": DecodeSpec("decode_swa_s16", 16, 1024, 32768, 64, 8, 128, 4096, 4096,
                                 1.0, 3),
}


def scaled(spec, **kw):
    """Same workload with some sizes replaced (for small parity cases)."""
    return replace(spec, **kw)


def _normal_bf16(gen, shape, device, std=1.0, chunk=1 << 28):
    """bf16 N(0, std) drawn in fp32 chunks (bounds the fp32 temporary)."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        tmp = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
        if std != 1.0:
            tmp.mul_(std)
        flat[s:e].copy_(tmp)
    return out


def _generator(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_prefill(spec: PrefillSpec, device="cpu"):
    g = _generator(device, spec.seed)
    B, T, Hq, Hkv, d = spec.B, spec.T, spec.Hq, spec.Hkv, spec.d
    C = Hkv * d
    q = _normal_bf16(g, (B, T, Hq, d), device)
    k_raw = _normal_bf16(g, (B, T, Hkv, d), device)
    v_raw = _normal_bf16(g, (B, T, Hkv, d), device)
    w_k = torch.randn((C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    w_v = torch.randn((C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    bias = torch.randn((Hq, spec.D_max + 1), generator=g, device=device,
                       dtype=torch.float32) * spec.bias_std
    return dict(q=q, k_raw=k_raw, v_raw=v_raw, w_k=w_k, w_v=w_v, bias=bias)


def make_decode(spec: DecodeSpec, device="cpu", extra_blocks: int = 0):
    """Decode step inputs.  ``seq_lens`` already count the n_new tokens that the
    sconv append writes; the cache holds N(0, 1) post-sconv rows for every
    allocated slot (the append overwrites the new tokens' slots)."""
    g = _generator(device, spec.seed)
    S, Hq, Hkv, d, n_new = spec.S, spec.Hq, spec.Hkv, spec.d, spec.n_new
    C = Hkv * d
    # one query per sequence, or the n_new newest tokens all as queries
    # (multi-token decode: the draft tokens of speculative decoding)
    q = _normal_bf16(g, (S, Hq, d) if n_new == 1 else (S, n_new, Hq, d), device)
    k_new = _normal_bf16(g, (S, n_new, Hkv, d), device)
    v_new = _normal_bf16(g, (S, n_new, Hkv, d), device)
    w_k = torch.randn((C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    w_v = torch.randn((C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    bias = torch.randn((Hq, spec.D_max + 1), generator=g, device=device,
                       dtype=torch.float32) * spec.bias_std
    k_state = _normal_bf16(g, (S, 3, C), device)
    v_state = _normal_bf16(g, (S, 3, C), device)
    if spec.L_min == spec.L_max:
        seq_lens = torch.full((S,), spec.L_min, dtype=torch.int32, device=device)
    else:
        seq_lens = torch.randint(spec.L_min, spec.L_max + 1, (S,), generator=g,
                                 device=device, dtype=torch.int64).to(torch.int32)
    blocks_per_seq = (seq_lens.to(torch.int64) + BLOCK - 1) // BLOCK
    max_blocks = int(blocks_per_seq.max().item())
    total = int(blocks_per_seq.sum().item()) + extra_blocks
    perm = torch.randperm(total, generator=g, device=device).to(torch.int32)
    block_table = torch.zeros((S, max_blocks), dtype=torch.int32, device=device)
    off = 0
    for s in range(S):
        nb = int(blocks_per_seq[s].item())
        block_table[s, :nb] = perm[off:off + nb]
        off += nb
    k_cache = _normal_bf16(g, (total, Hkv, BLOCK, d), device)
    v_cache = _normal_bf16(g, (total, Hkv, BLOCK, d), device)
    return dict(q=q, k_new=k_new, v_new=v_new, w_k=w_k, w_v=w_v, bias=bias,
                k_state=k_state, v_state=v_state, seq_lens=seq_lens,
                block_table=block_table, k_cache=k_cache, v_cache=v_cache)


def kv_bytes_read(spec: DecodeSpec, seq_lens) -> int:
    """Post-sconv K+V bytes inside each sequence's window or context (for
    n_new query tokens, the union of their windows: W + n_new - 1 keys)."""
    W = spec.window
    tot = 0
    for L in seq_lens.tolist():
        n = min(L, W + spec.n_new - 1) if W > 0 else L
        tot += n
    return tot * spec.Hkv * spec.d * 2 * 2


def make_chunk(spec: ChunkSpec, device="cpu"):
    """Chunked-prefill step inputs: packed chunk queries q [B*chunk, Hq, d] with
    row offsets cu_q, the chunk's raw keys/values [B, chunk, Hkv, d], taps,
    bias, sconv states, and a paged cache whose prefix slots hold N(0, 1)
    post-sconv rows (the append overwrites the chunk's slots).  With no
    prefix the sconv states are zero."""
    g = _generator(device, spec.seed)
    B, Hq, Hkv, d, n = spec.B, spec.Hq, spec.Hkv, spec.d, spec.chunk
    C = Hkv * d
    q = _normal_bf16(g, (B * n, Hq, d), device)
    k_new = _normal_bf16(g, (B, n, Hkv, d), device)
    v_new = _normal_bf16(g, (B, n, Hkv, d), device)
    w_k = torch.randn((C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    w_v = torch.randn((C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    bias = torch.randn((Hq, spec.D_max + 1), generator=g, device=device,
                       dtype=torch.float32) * spec.bias_std
    k_state = _normal_bf16(g, (B, 3, C), device)
    v_state = _normal_bf16(g, (B, 3, C), device)
    if spec.prefix == 0:  # an empty sequence has zero sconv history
        k_state.zero_()
        v_state.zero_()
    L = spec.prefix + n
    nb = (L + BLOCK - 1) // BLOCK
    perm = torch.randperm(B * nb, generator=g, device=device).to(torch.int32)
    block_table = perm.reshape(B, nb).contiguous()
    k_cache = _normal_bf16(g, (B * nb, Hkv, BLOCK, d), device)
    v_cache = _normal_bf16(g, (B * nb, Hkv, BLOCK, d), device)
    seq_lens = torch.full((B,), L, dtype=torch.int32, device=device)
    cu_q = torch.arange(0, (B + 1) * n, n, dtype=torch.int32, device=device)
    return dict(q=q, cu_q=cu_q, k_new=k_new, v_new=v_new, w_k=w_k, w_v=w_v, bias=bias,
                k_state=k_state, v_state=v_state, seq_lens=seq_lens, block_table=block_table,
                k_cache=k_cache, v_cache=v_cache)


def make_sconv_out(spec: SconvOutSpec, device="cpu"):
    g = _generator(device, spec.seed)
    x = _normal_bf16(g, (spec.B, spec.T, spec.C), device)
    w = torch.randn((spec.C, 4), generator=g, device=device, dtype=torch.float32) * 0.5
    state = _normal_bf16(g, (spec.B, 3, spec.C), device)
    return dict(x=x, w=w, state=state)

