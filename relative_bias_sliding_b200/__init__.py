"""Inkling decoder attention layer for NVIDIA B200 (sm_100a).

The layer: a causal depthwise window-4 short convolution over keys and values,
then grouped-query attention at head size 128 with a learned relative-position
bias added to the logits, sliding-window or full causal.  The compute runs in
libinkling.so (hand-written CUDA, C ABI in include/inkling.h); ``binding``
marshals torch tensors into it and ``inputs`` draws seeded synthetic inputs.
"""
from .binding import (  # noqa: F401
    InklingError,
    attn_decode,
    attn_decode_static,
    attn_prefill,
    attn_prefill_paged,
    decode_num_splits,
    decode_workspace_bytes,
    load_library,
    prefill_workspace_bytes,
    sconv_kv,
    sconv_out,
    sconv_out_sharded,
)

__all__ = ["attn_prefill", "attn_prefill_paged", "attn_decode", "attn_decode_static", "sconv_kv", "decode_num_splits",
           "decode_workspace_bytes", "prefill_workspace_bytes", "load_library", "InklingError",
           "sconv_out", "sconv_out_sharded"]
