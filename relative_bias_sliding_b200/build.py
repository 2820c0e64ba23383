"""Build libinkling.so (all CUDA sources, sm_100a) next to this file.

Run ``python -m relative_bias_sliding_b200.build`` or call ``build()``.  nvcc
cross-compiles for sm_100a on a machine without a GPU.  The CUDA runtime is
linked statically so the library does not depend on which libcudart the host
process loaded; the driver API is reached through cudaGetDriverEntryPoint.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libinkling.so")
SOURCES = ["api.cu", "sconv_kv.cu", "attn_decode.cu", "attn_prefill.cu", "attn_prefill_pair.cu",
           "attn_prefill_paged.cu", "sconv_out.cu", "attn_decode_mq.cu", "sconv_shard.cu"]
HEADERS = ["common.cuh", "prefill_common.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libinkling")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "inkling.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = nvcc_path()
    outdir = os.path.join(ROOT, "_build")
    os.makedirs(outdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(outdir, src.replace(".cu", ".o"))
        cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
               "-I", os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
