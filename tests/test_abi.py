"""The C-ABI library loads, exports every entry point include/inkling.h
declares, its parameter structs match the ctypes mirrors byte for byte, and
host-side validation rejects bad arguments before touching a device (CPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from relative_bias_sliding_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "inkling.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(inkling_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(binding.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (inkling_\w+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)


def test_struct_layouts_match_header(tmp_path):
    src = tmp_path / "sizes.c"
    src.write_text(f"""
#include <stddef.h>
#include <stdio.h>
#include "{HEADER}"
#define F(S, m) printf(#S " " #m " %zu\\n", offsetof(S, m));
int main(void) {{
  printf("sconv %zu\\nprefill %zu\\ndecode %zu\\npaged %zu\\n", sizeof(inkling_sconv_params),
         sizeof(inkling_prefill_params), sizeof(inkling_decode_params),
         sizeof(inkling_prefill_paged_params));
  F(inkling_sconv_params, num_blocks) F(inkling_prefill_params, d_max)
  F(inkling_prefill_params, k_cache) F(inkling_prefill_params, max_blocks)
  F(inkling_prefill_params, v_state) F(inkling_prefill_params, path)
  F(inkling_prefill_params, workspace) F(inkling_prefill_params, workspace_bytes)
  F(inkling_decode_params, num_splits) F(inkling_decode_params, status)
  F(inkling_decode_params, q_len) F(inkling_prefill_paged_params, cu_q)
  F(inkling_prefill_paged_params, max_q) F(inkling_prefill_paged_params, d_max)
  printf("sconv_out %zu\\n", sizeof(inkling_sconv_out_params));
  F(inkling_sconv_out_params, y) F(inkling_sconv_out_params, channels)
  printf("sharded %zu\\n", sizeof(inkling_sconv_out_sharded_params));
  F(inkling_sconv_out_sharded_params, state) F(inkling_sconv_out_sharded_params, n_ranks)
  F(inkling_sconv_out_sharded_params, channels)
  printf("paths %d%d%d\\n", INKLING_PREFILL_AUTO, INKLING_PREFILL_FUSED, INKLING_PREFILL_TWO_PASS);
  printf("min_t %d\\n", INKLING_PREFILL_TWO_PASS_MIN_T);
  printf("min_tokens %d\\n", INKLING_PREFILL_TWO_PASS_MIN_TOKENS);
  return 0;
}}""")
    exe = tmp_path / "sizes"
    subprocess.run(["gcc", str(src), "-o", str(exe)], check=True)
    out = dict(l.rsplit(" ", 1) for l in subprocess.run([str(exe)], capture_output=True,
                                                         text=True).stdout.splitlines())
    assert int(out["sconv"]) == ctypes.sizeof(binding.SconvParams)
    assert int(out["prefill"]) == ctypes.sizeof(binding.PrefillParams)
    assert int(out["decode"]) == ctypes.sizeof(binding.DecodeParams)
    assert int(out["inkling_sconv_params num_blocks"]) == binding.SconvParams.num_blocks.offset
    assert int(out["inkling_prefill_params d_max"]) == binding.PrefillParams.d_max.offset
    for m in ("k_cache", "max_blocks", "v_state", "path", "workspace", "workspace_bytes"):
        assert int(out["inkling_prefill_params " + m]) == getattr(binding.PrefillParams, m).offset
    assert int(out["inkling_decode_params num_splits"]) == binding.DecodeParams.num_splits.offset
    assert int(out["inkling_decode_params status"]) == binding.DecodeParams.status.offset
    assert int(out["inkling_decode_params q_len"]) == binding.DecodeParams.q_len.offset
    P = binding.PrefillPagedParams
    assert int(out["paged"]) == ctypes.sizeof(P)
    assert int(out["inkling_prefill_paged_params cu_q"]) == P.cu_q.offset
    assert int(out["inkling_prefill_paged_params max_q"]) == P.max_q.offset
    assert int(out["inkling_prefill_paged_params d_max"]) == P.d_max.offset
    O = binding.SconvOutParams
    assert int(out["sconv_out"]) == ctypes.sizeof(O)
    assert int(out["inkling_sconv_out_params y"]) == O.y.offset
    assert int(out["inkling_sconv_out_params channels"]) == O.channels.offset
    P = binding.PREFILL_PATHS
    assert out["paths"] == f"{P['auto']}{P['fused']}{P['two_pass']}"
    assert int(out["min_t"]) == binding.INKLING_PREFILL_TWO_PASS_MIN_T
    assert int(out["min_tokens"]) == binding.INKLING_PREFILL_TWO_PASS_MIN_TOKENS
    H = binding.SconvOutShardedParams
    assert int(out["sharded"]) == ctypes.sizeof(H)
    for m in ("state", "n_ranks", "channels"):
        assert int(out["inkling_sconv_out_sharded_params " + m]) == getattr(H, m).offset


def test_sharded_sconv_validation_rejects_before_launch(lib):
    # argument checks come before any device access (addresses never read)
    f = lib.inkling_sconv_out_sharded
    fake = [ctypes.c_void_p((1 << 20) + (i << 24)) for i in range(4)]
    xs = (ctypes.c_void_p * 2)(fake[0], fake[1])
    ys = (ctypes.c_void_p * 2)(fake[2], fake[3])
    p = binding.SconvOutShardedParams(xs, ys, fake[0], None, 2, 0, 1, 16, 256)
    p.n_ranks = 9
    assert f(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    p.n_ranks, p.rank = 2, 2
    assert f(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    p.rank, p.channels = 1, 24   # not a multiple of 8 * n_ranks
    assert f(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    p.channels = 256
    p.y_parts = (ctypes.c_void_p * 2)(fake[2], fake[1])   # y_parts[1] is x_parts[1]
    assert f(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"overlaps" in lib.inkling_last_error()
    p.seq_len = 0
    assert f(ctypes.byref(p), None) == binding.INKLING_OK   # empty: no-op


def test_workspace_bytes(lib):
    f = lib.inkling_attn_decode_workspace_bytes
    assert f(64, 64, 4) == 64 * 64 * 4 * 130 * 4
    assert f(1, 64, 148) == 64 * 148 * 130 * 4
    assert f(3, 8, 1) == 16
    assert f(-1, 8, 2) == 0 and f(3, 0, 2) == 0 and f(3, 8, 0) == 0 and f(3, 8, 1025) == 0


def test_prefill_workspace_bytes(lib):
    """The two-pass prefill's scratch: post-sconv K and V of ceil(T/128) blocks
    per sequence; none for the fused path, with a cache, or below the
    automatic path's thresholds (B*T >= 2048 tokens and T >= 512)."""
    f = lib.inkling_attn_prefill_workspace_bytes
    p = binding.PrefillParams()
    p.batch, p.seq_len, p.num_q_heads, p.num_kv_heads, p.head_dim = 4, 8192, 64, 8, 128
    assert f(ctypes.byref(p)) == 2 * 4 * 64 * 8 * 128 * 128 * 2  # auto, 8192 tokens
    p.path = binding.PREFILL_PATHS["fused"]
    assert f(ctypes.byref(p)) == 0
    p.path, p.seq_len = binding.PREFILL_PATHS["auto"], 511
    assert f(ctypes.byref(p)) == 0  # T below 512: the automatic path fuses
    p.seq_len = 512
    assert f(ctypes.byref(p)) == 2 * 4 * 4 * 8 * 128 * 128 * 2  # B*T = 2048
    p.batch, p.seq_len = 1, 2047
    assert f(ctypes.byref(p)) == 0  # B*T below 2048
    p.seq_len = 2048
    assert f(ctypes.byref(p)) == 2 * 1 * 16 * 8 * 128 * 128 * 2
    p.batch = 4
    p.path, p.seq_len, p.batch = binding.PREFILL_PATHS["two_pass"], 300, 3  # ragged: 3 blocks
    assert f(ctypes.byref(p)) == 2 * 3 * 3 * 8 * 128 * 128 * 2
    p.k_cache = ctypes.c_void_p(1 << 20)
    assert f(ctypes.byref(p)) == 0  # the cache is the scratch
    p.k_cache, p.seq_len = None, 0
    assert f(ctypes.byref(p)) == 0
    assert f(None) == 0
    assert binding.INKLING_PREFILL_TWO_PASS_MIN_T == 512
    assert binding.INKLING_PREFILL_TWO_PASS_MIN_TOKENS == 2048


def test_prefill_path_validation_rejects_before_launch(lib):
    fake = ctypes.c_void_p(1 << 20)
    p = binding.PrefillParams()
    p.batch, p.seq_len, p.num_q_heads, p.num_kv_heads, p.head_dim = 1, 4096, 8, 1, 128
    for f in ("q", "k_raw", "v_raw", "w_k", "w_v", "bias", "out"):
        setattr(p, f, fake)
    p.path = 3
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"path" in lib.inkling_last_error()
    p.path = binding.PREFILL_PATHS["two_pass"]
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"workspace" in lib.inkling_last_error()
    p.workspace, p.workspace_bytes = fake, 2 * 32 * 128 * 128 * 2 - 16  # one row short
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"workspace" in lib.inkling_last_error()
    p.workspace = ctypes.c_void_p((1 << 20) + 8)
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"16-byte" in lib.inkling_last_error()
    p.workspace, p.workspace_bytes, p.seq_len = fake, 1 << 40, (1 << 20) + 1
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_UNSUPPORTED


def test_host_validation_rejects_before_launch(lib):
    # none of these reach the device: they fail argument checks first
    p = binding.PrefillParams()
    p.batch, p.seq_len, p.num_q_heads, p.num_kv_heads, p.head_dim = 1, 16, 8, 1, 64
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_UNSUPPORTED
    assert b"head_dim" in lib.inkling_last_error()
    p.head_dim, p.num_q_heads, p.num_kv_heads = 128, 6, 4
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    p.num_q_heads = 8
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID  # NULLs
    p.batch = 0
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_OK  # empty: no-op
    assert lib.inkling_attn_prefill(None, None) == binding.INKLING_ERR_INVALID

    # the optional cache fill: argument checks come before any device access
    # (the addresses below are never dereferenced)
    fake = ctypes.c_void_p(1 << 20)
    p.batch = 1
    for f in ("q", "k_raw", "v_raw", "w_k", "w_v", "bias", "out"):
        setattr(p, f, fake)
    p.k_cache = fake
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"together" in lib.inkling_last_error()
    p.v_cache, p.block_table, p.max_blocks, p.num_blocks = fake, fake, 0, 4
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    p.seq_len, p.max_blocks = 300, 2
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"max_blocks * 128" in lib.inkling_last_error()
    p.max_blocks, p.k_state = 3, fake
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"k_state and v_state" in lib.inkling_last_error()
    p.v_state = ctypes.c_void_p((1 << 20) + 8)
    assert lib.inkling_attn_prefill(ctypes.byref(p), None) == binding.INKLING_ERR_INVALID
    assert b"16-byte" in lib.inkling_last_error()

    d = binding.DecodeParams()
    d.num_seqs, d.num_q_heads, d.num_kv_heads, d.head_dim = 2, 64, 4, 128
    d.max_blocks, d.num_blocks = 4, 8
    assert lib.inkling_attn_decode(ctypes.byref(d), None, 0, None) == binding.INKLING_ERR_UNSUPPORTED
    d.num_kv_heads = 8
    assert lib.inkling_attn_decode(ctypes.byref(d), None, 0, None) == binding.INKLING_ERR_INVALID
    d.num_splits = 2000
    assert lib.inkling_attn_decode(ctypes.byref(d), None, 0, None) == binding.INKLING_ERR_INVALID

    s = binding.SconvParams()
    s.num_seqs, s.n_new, s.num_kv_heads, s.head_dim, s.max_blocks, s.num_blocks = 1, 0, 1, 128, 1, 1
    assert lib.inkling_sconv_kv(ctypes.byref(s), None) == binding.INKLING_ERR_INVALID
    s.n_new = 1
    assert lib.inkling_sconv_kv(ctypes.byref(s), None) == binding.INKLING_ERR_INVALID  # NULLs


def test_product_path_does_not_import_oracle():
    # the binding, the build script and the kernels never reference the oracle
    pkg = os.path.join(ROOT, "relative_bias_sliding_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "liboracle" not in text and "oracle.c" not in text, f
