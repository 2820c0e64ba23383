#!/usr/bin/env python3
"""Benchmark of the Inkling decoder attention layer on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill: the sliding-window prefill workload (B=4, T=8192, Hq=64, Hkv=8,
    d=128, window 4096) through inkling_attn_prefill on its automatic path
    (at this length two kernels: the sconv of all keys/values written once
    into a preallocated workspace in the paged layout, then the paged
    prefill kernel; the fused one-kernel path is timed beside it);
  * decode: the sliding-window decode workload (64 sequences, lengths uniform
    in [1024, 32768], window 4096, paged 128-token blocks) through
    inkling_sconv_kv + inkling_attn_decode.
The headline ``value`` is prefill TFLOP/s (allowed (i, j) pairs x 4 d Hq B);
the decode step is reported beside it in KV GB/s (post-sconv K+V bytes inside
each window).  ``--workload`` picks any single workload instead.

Launch: ``python bench.py --gpus N --steps K --warmup W`` (N > 1 under
torch.distributed.run: every rank runs the same workload on its own GPU, no
data-path collective, weak scaling; times are max over ranks).
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill TFLOP/s and decode KV GB/s on 1 B200, as % of BF16/HBM roofline"
DEFAULT_PREFILL = "prefill_swa_b4_t8192"
DEFAULT_DECODE = "decode_swa_s64"
# the same sliding-window prefill shape through the paged cache: sconv append
# of all keys/values, then the paged prefill (timed after the main step)
DEFAULT_VIA_CACHE = "prefill_paged_swa_b4_t8192"
# the layer's other workloads, each timed after the step with its own roofline
# and oracle timing: the tiny and the 32k full-causal prefill; multi-token
# decode (9 draft tokens); 1M-token full-attention decode at batch 1 and 8
EXTRA_PREFILL = ["prefill_tiny_b1_t256", "prefill_full_b1_t32768"]
EXTRA_DECODE = ["decode_mtp9_swa_s64", "decode_full_1m_b1", "decode_full_1m_b8"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of the current kernels on the workload itself (one launch after
# 3 warm-up launches; profiles/ holds the summaries and commands).  Remove an
# entry when its kernel changes until it is captured again.
MEASURED_TRAFFIC = {
    # the prefill call's dominant kernel: the paged kernel on the two-pass path,
    # the pair kernel on the fused one (" fused")
    "prefill_swa_b4_t8192": 676_627_968 + 496_061_952,
    "prefill_swa_b4_t8192 fused": 680_339_712 + 501_876_992,
    "prefill_paged_swa_b4_t8192": 676_296_960 + 498_352_896,
    "prefill_chunked_swa_b4_c2048": 237_998_336 + 99_810_560,
    "decode_swa_s64": 1_080_809_216 + 3_773_440,
    "decode_mtp9_swa_s64": 1_089_955_584 + 8_819_968,
}


# ------------------------------------------------------------ distributed --

def dist_env():
    """(rank, world, local_rank) from the torch.distributed.run environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(dist, values, device="cpu"):
    """Element-wise max of a list of floats over all ranks (timing only)."""
    import torch
    if dist is None:
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, log_dir=None):
        # the raw samples go to <log_dir>/clocks_gpu<i>.csv when a directory
        # is given, else to a temporary file
        self.gpu = gpu_index
        self.proc = None
        if log_dir:
            self.path = os.path.join(log_dir, f"clocks_gpu{gpu_index}.csv")
        else:
            self.path = os.path.join(tempfile.gettempdir(), f"inkling_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ peaks --

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_roofline(achieved, kernel, traffic=None, clocks=None):
    """Roofline object of a tensor-bound kernel.  The peak is the burst cuBLAS
    bf16 figure: the kernels here run at the maximum SM clock without the power
    cap (the `clocks` of the same line show it), so the burst figure, the
    higher of the two measured peaks, is the one they are held to; the
    fraction of the sustained (power-capped) figure is given beside it."""
    peaks, src = load_peaks()
    burst = peaks["bf16_tflops"]
    sus = peaks.get("bf16_tflops_sustained", burst)
    note = f"{src} bf16_tflops (burst)"
    if clocks:
        note += (f"; kernel timed at median {clocks.get('sm_mhz')} MHz of max "
                 f"{clocks.get('sm_max_mhz')}, reasons {clocks.get('reasons')}")
    return {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": burst,
            "unit": "TFLOP/s", "frac": achieved / burst, "traffic": traffic, "peak_source": note,
            "frac_of_sustained": achieved / sus, "sustained_peak": sus}


def hbm_roofline(achieved, kernel, traffic=None):
    peaks, src = load_peaks()
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": f"{src} hbm_gbs"}


# ----------------------------------------------------------- GPU workload --

class PrefillStep:
    """One prefill call on the automatic path (two-pass from 2048 tokens per call:
    sconv into a preallocated workspace, then the paged prefill kernel; fused
    below), plus the fused kernel and the cache-filling variants of the same
    call, and the two passes as separate public calls for their timings."""

    def __init__(self, spec, device, path="auto"):
        import torch
        import relative_bias_sliding_b200 as ink
        from relative_bias_sliding_b200.inputs import make_prefill
        self.spec = spec
        self.t = make_prefill(spec, device=device)
        self.out = torch.empty_like(self.t["q"])
        self.flops = spec.flops
        self.path_arg = path
        nbytes = ink.prefill_workspace_bytes(spec.B, spec.T, spec.Hq, spec.Hkv, path=path)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device) if nbytes else None
        self.two_pass = nbytes > 0
        self.launches = 2 if self.two_pass else 1
        self.path = "two_pass" if self.two_pass else "fused"
        self.kernel = "attn_prefill_paged_kernel" if self.two_pass else "attn_prefill_pair_kernel"

    def run(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.attn_prefill(t["q"], t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], t["bias"],
                         window=self.spec.window, out=self.out, stream=stream,
                         path=self.path_arg, workspace=self.ws)

    def run_fused(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.attn_prefill(t["q"], t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], t["bias"],
                         window=self.spec.window, out=self.out, stream=stream, path="fused")

    def add_parts(self, device):
        """Buffers for the two passes as separate public calls: the sconv
        append of all T tokens into a cache in the scratch's block order
        (sequence b on blocks b*nb ...), then the paged prefill of every
        sequence as one chunk of T rows."""
        import torch
        B, T, Hq, Hkv = self.spec.B, self.spec.T, self.spec.Hq, self.spec.Hkv
        nb = (T + 127) // 128
        self.p_bt = torch.arange(B * nb, dtype=torch.int32, device=device).reshape(B, nb)
        self.p_kc = torch.zeros((B * nb, Hkv, 128, 128), dtype=torch.bfloat16, device=device)
        self.p_vc = torch.zeros_like(self.p_kc)
        self.p_ks = torch.zeros((B, 3, Hkv * 128), dtype=torch.bfloat16, device=device)
        self.p_vs = torch.zeros_like(self.p_ks)
        self.p_lens = torch.full((B,), T, dtype=torch.int32, device=device)
        self.p_cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=device)

    def run_part_sconv(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.sconv_kv(t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], self.p_ks, self.p_vs,
                     self.p_kc, self.p_vc, self.p_bt, self.p_lens, stream=stream)

    def run_part_attn(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t, sp = self.t, self.spec
        rows = sp.B * sp.T
        ink.attn_prefill_paged(t["q"].view(rows, sp.Hq, sp.d), self.p_cu, self.p_kc, self.p_vc,
                               self.p_bt, self.p_lens, t["bias"], window=sp.window, max_q=sp.T,
                               out=self.out.view(rows, sp.Hq, sp.d), stream=stream)

    def add_cache(self, device):
        """Paged cache, block table and sconv states for the cache-filling
        variant of the same prefill (blocks in a random order)."""
        import torch
        B, T, Hkv = self.spec.B, self.spec.T, self.spec.Hkv
        nb = (T + 127) // 128
        g = torch.Generator(device=device).manual_seed(self.spec.seed + 100)
        self.bt = torch.randperm(B * nb, generator=g, device=device).to(torch.int32).reshape(B, nb)
        self.kc = torch.zeros((B * nb, Hkv, 128, 128), dtype=torch.bfloat16, device=device)
        self.vc = torch.zeros_like(self.kc)
        self.ks = torch.zeros((B, 3, Hkv * 128), dtype=torch.bfloat16, device=device)
        self.vs = torch.zeros_like(self.ks)

    def run_fill(self, stream=None, path="auto"):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.attn_prefill(t["q"], t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], t["bias"],
                         window=self.spec.window, out=self.out, stream=stream, k_cache=self.kc,
                         v_cache=self.vc, block_table=self.bt, k_state=self.ks, v_state=self.vs,
                         path=path)

    def run_fill_fused(self, stream=None):
        self.run_fill(stream, path="fused")


class DecodeStep:
    def __init__(self, spec, device):
        import torch
        import relative_bias_sliding_b200 as ink
        from relative_bias_sliding_b200.inputs import make_decode, kv_bytes_read
        self.spec = spec
        self.t = make_decode(spec, device=device)
        t = self.t
        self.out = torch.empty_like(t["q"])
        self.splits = ink.decode_num_splits(t["q"], t["k_cache"], t["v_cache"],
                                            t["block_table"], t["seq_lens"], t["bias"],
                                            window=spec.window)
        rows = spec.S * (t["q"].shape[1] if t["q"].dim() == 4 else 1)  # (sequence, token) rows
        nbytes = max(16, ink.decode_workspace_bytes(rows, spec.Hq, self.splits))
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.kv_bytes = kv_bytes_read(spec, t["seq_lens"].cpu())
        self.cache_bytes = 2 * t["k_cache"].numel() * t["k_cache"].element_size()
        self.launches = 2 + (1 if self.splits > 1 else 0)

    def run_append(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.sconv_kv(t["k_new"], t["v_new"], t["w_k"], t["w_v"], t["k_state"], t["v_state"],
                     t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"], stream=stream)

    def run_attn(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        # num_splits 0: the library's own plan, with the workspace sized for
        # the split count it reports
        ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                        t["bias"], window=self.spec.window, out=self.out, workspace=self.ws,
                        num_splits=0, stream=stream)

    def run(self, stream=None):
        self.run_append(stream)
        self.run_attn(stream)


class ChunkStep:
    """Chunked prefill step: sconv append of every sequence's chunk, then the
    chunk rows over the paged cache."""

    def __init__(self, spec, device):
        import torch
        from relative_bias_sliding_b200.inputs import make_chunk
        self.spec = spec
        self.t = make_chunk(spec, device=device)
        self.out = torch.empty_like(self.t["q"])
        self.flops = spec.flops
        self.launches = 2
        mib = lambda x: x.numel() * x.element_size() / 2**20
        cache = mib(self.t["k_cache"]) + mib(self.t["v_cache"])
        self.l2_note = (f"inputs larger than L2 (q {mib(self.t['q']):.0f} MiB, "
                        f"K/V cache {cache:.0f} MiB)")

    def run_append(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.sconv_kv(t["k_new"], t["v_new"], t["w_k"], t["w_v"], t["k_state"], t["v_state"],
                     t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"], stream=stream)

    def run_attn(self, stream=None):
        import relative_bias_sliding_b200 as ink
        t = self.t
        ink.attn_prefill_paged(t["q"], t["cu_q"], t["k_cache"], t["v_cache"], t["block_table"],
                               t["seq_lens"], t["bias"], window=self.spec.window,
                               max_q=self.spec.chunk, out=self.out, stream=stream)


def timed_loop(steps, fns, stream):
    """Run ``steps`` iterations of the callables in order on ``stream``; return
    per-callable mean milliseconds (CUDA events recorded on that stream)."""
    import torch
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in fns] for _ in range(steps)]
    for k in range(steps):
        for (a, b), fn in zip(evs[k], fns):
            a.record(stream)
            fn(stream)
            b.record(stream)
    stream.synchronize()
    return [sum(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(steps)) / steps
            for i in range(len(fns))]


def pipelined_steps(steps, h2d, compute, d2h, stream):
    """Time ``steps`` end-to-end steps as a server runs them: step i's inputs
    copy in (pinned host -> device, own stream) while step i-1 computes and
    step i-2's result copies out (device -> pinned host, own stream).  Device
    buffers are double-buffered by step parity; events order each buffer's
    reuse.  Every step's copies fall inside the timed region, which starts
    before the first copy-in and ends after the last copy-out.  Returns mean
    milliseconds per step."""
    import torch
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def issue(i):
        b = i & 1
        if i >= 2:
            s_in.wait_event(comp_done[b])  # step i-2 has finished reading inputs[b]
        h2d(b, s_in)
        in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        if i >= 2:
            stream.wait_event(out_done[b])  # step i-2's result has left outputs[b]
        compute(b, stream)
        comp_done[b].record(stream)
        s_out.wait_event(comp_done[b])
        d2h(b, s_out)
        out_done[b].record(s_out)

    for i in range(2):  # warm-up through both buffers
        issue(i)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    for i in range(steps):
        issue(i)
    stream.wait_event(out_done[(steps - 1) & 1])
    z.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(z) / steps


def e2e_prefill(step, steps, stream):
    """Same prefill through the public API with host buffers: pinned host ->
    device copies of the step's inputs, the call, and the output read back,
    pipelined across steps (pipelined_steps)."""
    import torch
    t = step.t
    host = {k: t[k].cpu().pin_memory() for k in ("q", "k_raw", "v_raw")}
    out_h = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    dev = [{k: torch.empty_like(t[k]) for k in host} for _ in range(2)]
    outs = [step.out, torch.empty_like(step.out)]
    import relative_bias_sliding_b200 as ink

    def h2d(b, s):
        with torch.cuda.stream(s):
            for k in host:
                dev[b][k].copy_(host[k], non_blocking=True)

    def compute(b, s):
        ink.attn_prefill(dev[b]["q"], dev[b]["k_raw"], dev[b]["v_raw"], t["w_k"], t["w_v"],
                         t["bias"], window=step.spec.window, out=outs[b], stream=s,
                         path=step.path_arg, workspace=step.ws)  # calls in order on one stream

    def d2h(b, s):
        with torch.cuda.stream(s):
            out_h.copy_(outs[b], non_blocking=True)

    ms = pipelined_steps(steps, h2d, compute, d2h, stream)
    h2d_bytes = sum(v.numel() * v.element_size() for v in host.values())
    return ms, h2d_bytes, out_h.numel() * out_h.element_size()


def e2e_decode(step, steps, stream):
    """Decode step through the public API with host buffers for the per-step
    inputs (queries, new raw keys/values, lengths, block table), pipelined
    across steps (pipelined_steps); the caches and sconv states stay resident
    as the layer's state."""
    import torch
    t = step.t
    names = ("q", "k_new", "v_new", "seq_lens", "block_table")
    host = {k: t[k].cpu().pin_memory() for k in names}
    out_h = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    dev = [{k: torch.empty_like(t[k]) for k in names} for _ in range(2)]
    outs = [step.out, torch.empty_like(step.out)]
    import relative_bias_sliding_b200 as ink

    def h2d(b, s):
        with torch.cuda.stream(s):
            for k in names:
                dev[b][k].copy_(host[k], non_blocking=True)

    def compute(b, s):
        d = dev[b]
        ink.sconv_kv(d["k_new"], d["v_new"], t["w_k"], t["w_v"], t["k_state"], t["v_state"],
                     t["k_cache"], t["v_cache"], d["block_table"], d["seq_lens"], stream=s)
        ink.attn_decode(d["q"], t["k_cache"], t["v_cache"], d["block_table"], d["seq_lens"],
                        t["bias"], window=step.spec.window, out=outs[b], workspace=step.ws,
                        num_splits=0, stream=s)

    def d2h(b, s):
        with torch.cuda.stream(s):
            out_h.copy_(outs[b], non_blocking=True)

    ms = pipelined_steps(steps, h2d, compute, d2h, stream)
    h2d_bytes = sum(v.numel() * v.element_size() for v in host.values())
    return ms, h2d_bytes, out_h.numel() * out_h.element_size()


# ------------------------------------------------------------ CPU oracle --

def oracle_prefill_sample(spec, seconds, seed=0):
    """Time the oracle on a bounded row sample of a prefill workload; returns
    (TFLOP/s, description, threads)."""
    import numpy as np
    import torch
    import oracle
    from relative_bias_sliding_b200.inputs import make_prefill
    t = make_prefill(spec, device="cpu")
    u = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    rng = np.random.default_rng(seed)
    W, T = spec.window, spec.T
    per_row = lambda i: (min(i + 1, W) if W > 0 else i + 1)
    # calibrate on a small batch, then size the sample to about `seconds`
    n = 64
    total_rows, total_flops, total_t = 0, 0, 0.0
    while True:
        b = rng.integers(0, spec.B, n)
        h = rng.integers(0, spec.Hq, n)
        i = rng.integers(0, T, n)
        rows = np.stack([b, h, i], 1).astype(np.int32)
        t0 = time.perf_counter()
        oracle.prefill_rows(u(t["q"]), u(t["k_raw"]), u(t["v_raw"]), t["w_k"].numpy(),
                            t["w_v"].numpy(), t["bias"].numpy(), W, spec.D_max, rows)
        dt = time.perf_counter() - t0
        total_t += dt
        total_rows += n
        total_flops += sum(4 * spec.d * per_row(int(x)) for x in i)
        if total_t >= seconds:
            break
        n = int(min(1 << 16, max(n * 2, n * (seconds - total_t) / max(dt, 1e-3))))
    desc = (f"{total_rows} random query rows of {spec.name} (sconv of all keys/values "
            f"included in every call), {total_t:.1f} s")
    return total_flops / total_t / 1e12, desc, oracle.num_threads()


def oracle_decode_sample(spec, seconds, seed=0):
    """Time the oracle's decode step (sconv append + attention) on whole
    sequences of a decode workload; returns (KV GB/s, description, threads)."""
    import numpy as np
    import torch
    import oracle
    from relative_bias_sliding_b200.inputs import make_decode, scaled
    sub = scaled(spec, S=min(spec.S, 8))
    t = make_decode(sub, device="cpu")
    u = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    kc, vc = u(t["k_cache"]).copy(), u(t["v_cache"]).copy()
    ks, vs = u(t["k_state"]).copy(), u(t["v_state"]).copy()
    bt, sl = t["block_table"].numpy(), t["seq_lens"].numpy()
    W = sub.window
    done_bytes, total_t, nseq = 0, 0.0, 0
    Q = sub.n_new
    # the sub-workload's sequences, over again until about `seconds` of oracle
    # time (a repeated append rewrites the same slot: the work is the same)
    for step in range(1 << 20):
        s = step % sub.S
        t0 = time.perf_counter()
        oracle.sconv_append(u(t["k_new"])[s:s + 1], ks[s:s + 1], t["w_k"].numpy(), kc,
                            bt[s:s + 1], sl[s:s + 1])
        oracle.sconv_append(u(t["v_new"])[s:s + 1], vs[s:s + 1], t["w_v"].numpy(), vc,
                            bt[s:s + 1], sl[s:s + 1])
        if Q == 1:
            pairs = np.array([[s, h] for h in range(sub.Hq)], np.int32)
            oracle.decode_rows(u(t["q"]), kc, vc, bt, sl, t["bias"].numpy(), W, sub.D_max, pairs)
        else:
            rows = np.array([[s, qi, h] for qi in range(Q) for h in range(sub.Hq)], np.int32)
            oracle.decode_mq_rows(u(t["q"]), kc, vc, bt, sl, t["bias"].numpy(), W, sub.D_max,
                                  rows)
        total_t += time.perf_counter() - t0
        L = int(sl[s])
        done_bytes += (min(L, W + Q - 1) if W > 0 else L) * sub.Hkv * sub.d * 4
        nseq += 1
        if total_t >= seconds:
            break
    desc = (f"{nseq} whole-sequence decode steps over {sub.S} sequences of {spec.name} "
            f"(all {sub.Hq} heads each, sconv append included), {total_t:.1f} s")
    return done_bytes / total_t / 1e9, desc, oracle.num_threads()


def oracle_decode_long_sample(dec):
    """Time the oracle's decode step on one whole sequence of a long-context
    decode workload whose cache lives on the device: sequence 0's blocks are
    copied to the host in order (K and V, 4 GiB at 1M tokens), then the sconv
    append of its new token and the attention of all its query heads run on
    the oracle.  Returns (KV GB/s, description, threads)."""
    import numpy as np
    import torch
    import oracle
    t, spec = dec.t, dec.spec
    u = lambda x: x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    L = int(t["seq_lens"][0])
    nb = (L + 127) // 128
    ids = t["block_table"][0, :nb].long()
    kc, vc = u(t["k_cache"][ids]).copy(), u(t["v_cache"][ids]).copy()
    ks, vs = u(t["k_state"][:1]).copy(), u(t["v_state"][:1]).copy()
    bt = np.arange(nb, dtype=np.int32)[None, :]
    sl = np.array([L], np.int32)
    q, kn, vn = u(t["q"][:1]), u(t["k_new"][:1]), u(t["v_new"][:1])
    wk, wv, bias = (t[k].cpu().numpy() for k in ("w_k", "w_v", "bias"))
    t0 = time.perf_counter()
    oracle.sconv_append(kn, ks, wk, kc, bt, sl)
    oracle.sconv_append(vn, vs, wv, vc, bt, sl)
    oracle.decode_rows(q, kc, vc, bt, sl, bias, spec.window, spec.D_max)
    dt = time.perf_counter() - t0
    keys = min(L, spec.window) if spec.window > 0 else L
    desc = (f"1 whole sequence of {spec.name} ({L} tokens, all {spec.Hq} heads, sconv append "
            f"included), {dt:.1f} s")
    return keys * spec.Hkv * spec.d * 4 / dt / 1e9, desc, oracle.num_threads()


def oracle_chunk_sample(spec, seconds, seed=0):
    """Time the oracle's chunked-prefill step (sconv append of one sequence's
    chunk, then its chunk rows over the paged cache, all heads) on a bounded
    sample of rows; returns (TFLOP/s, description, threads)."""
    import numpy as np
    import torch
    import oracle
    from relative_bias_sliding_b200.inputs import make_chunk, scaled
    sub = scaled(spec, B=1)
    t = make_chunk(sub, device="cpu")
    u = lambda x: x.contiguous().view(torch.int16).numpy().view(np.uint16)
    kc, vc = u(t["k_cache"]).copy(), u(t["v_cache"]).copy()
    ks, vs = u(t["k_state"]).copy(), u(t["v_state"]).copy()
    bt, sl = t["block_table"].numpy(), t["seq_lens"].numpy()
    n, W = sub.chunk, sub.window
    q = u(t["q"]).reshape(1, n, sub.Hq, sub.d)
    t0 = time.perf_counter()
    oracle.sconv_append(u(t["k_new"]), ks, t["w_k"].numpy(), kc, bt, sl)
    oracle.sconv_append(u(t["v_new"]), vs, t["w_v"].numpy(), vc, bt, sl)
    rng = np.random.default_rng(seed)
    done_flops, rows_done = 0, 0
    while time.perf_counter() - t0 < seconds:
        qi = rng.integers(0, n, 16)
        rows = np.array([[0, r, h] for r in qi for h in range(sub.Hq)], np.int32)
        oracle.decode_mq_rows(q, kc, vc, bt, sl, t["bias"].numpy(), W, sub.D_max, rows)
        for r in qi:
            i = sub.prefix + int(r)
            done_flops += 4 * sub.d * sub.Hq * (min(i + 1, W) if W > 0 else i + 1)
        rows_done += len(rows)
    total_t = time.perf_counter() - t0
    desc = (f"sconv append of one {n}-token chunk + {rows_done} (row, head) pairs of "
            f"{spec.name}, {total_t:.1f} s")
    return done_flops / total_t / 1e12, desc, oracle.num_threads()


def oracle_sconv_out_sample(spec, seconds, seed=0):
    """Time the oracle's sconv on slices of the output-sconv workload; returns
    (GB/s of x read + y written, description, threads)."""
    import numpy as np
    import torch
    import oracle
    from relative_bias_sliding_b200.inputs import make_sconv_out, scaled
    sub = scaled(spec, B=1, T=min(spec.T, 1024))
    t = make_sconv_out(sub, device="cpu")
    x = t["x"].contiguous().view(torch.int16).numpy().view(np.uint16)
    h = t["state"].contiguous().view(torch.int16).numpy().view(np.uint16)
    w = t["w"].numpy()
    t0, n = time.perf_counter(), 0
    while time.perf_counter() - t0 < seconds or n == 0:
        oracle.sconv(x, w, h)
        n += 1
    dt = time.perf_counter() - t0
    desc = f"{n} passes over a [1, {sub.T}, {sub.C}] slice of {spec.name}, {dt:.1f} s"
    return n * sub.bytes_moved / dt / 1e9, desc, oracle.num_threads()


# ------------------------------------------------------------------ main --

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=150)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None,
                    help="a single workload name from relative_bias_sliding_b200.inputs.WORKLOADS")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-log-dir", default=None,
                    help="keep the raw nvidia-smi clock samples in this directory")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--prefill-path", default="auto", choices=["auto", "fused", "two_pass"],
                    help="inkling_attn_prefill path of the timed prefill (default: the library's "
                         "automatic choice)")
    return ap.parse_args()


def run_reference(args):
    from relative_bias_sliding_b200.inputs import WORKLOADS, PrefillSpec, ChunkSpec, SconvOutSpec
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    name = args.workload or DEFAULT_PREFILL
    spec = WORKLOADS[name]
    vals = []
    descs = []
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for k in range(args.warmup + args.steps):
        if isinstance(spec, PrefillSpec):
            v, desc, thr = oracle_prefill_sample(spec, per_step, seed=k)
            unit = "TFLOP/s"
        elif isinstance(spec, ChunkSpec):
            v, desc, thr = oracle_chunk_sample(spec, per_step, seed=k)
            unit = "TFLOP/s"
        elif isinstance(spec, SconvOutSpec):
            v, desc, thr = oracle_sconv_out_sample(spec, per_step, seed=k)
            unit = "GB/s"
        else:
            v, desc, thr = oracle_decode_sample(spec, per_step, seed=k)
            unit = "GB/s"
        if k >= args.warmup:
            vals.append(v)
            descs.append(desc)
    value = statistics.mean(vals)
    # the same config as this bench's own arm: the default step is the
    # sliding-window prefill plus the sliding-window decode step
    workload = name if args.workload else f"{DEFAULT_PREFILL} + {DEFAULT_DECODE}"
    config = {"workload": workload, "parallelism": f"replica per GPU x{args.gpus}",
              "l2": "not applicable: the oracle runs on the host cores"}
    if isinstance(spec, PrefillSpec):
        config["prefill_path"] = "not applicable: the oracle computes every row directly"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": unit, "cores": thr, "kind": "oracle",
                             "sample": descs[0]},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    if not args.workload:
        # the decode half of the default step, as in this bench's own line
        dv, ddesc, dthr = oracle_decode_sample(WORKLOADS[DEFAULT_DECODE], per_step / 2)
        line["decode"] = {"workload": DEFAULT_DECODE, "value": dv, "unit": "GB/s",
                          "cpu_baseline": {"value": dv, "unit": "GB/s", "cores": dthr,
                                           "kind": "oracle", "sample": ddesc}}
    print(json.dumps(line), flush=True)
    return 0


def time_loop_only(args, fns, dist, device):
    """Warm up, then time ``args.steps`` passes over ``fns`` on one stream;
    per-callable mean ms, max over ranks."""
    import torch
    stream = torch.cuda.Stream(device)
    for _ in range(args.warmup):
        for f in fns:
            f(stream)
    stream.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    per_fn = timed_loop(args.steps, fns, stream)
    torch.cuda.synchronize()
    barrier(dist, device)
    return max_over_ranks(dist, per_fn, device)


def time_chunk(args, chk, dist, local, device, clocks_dir):
    """Warm up, then time ``args.steps`` chunk steps (append, paged prefill) on
    one stream; returns (step ms, append ms, attention ms) as the max over
    ranks, and the clock sampler."""
    import torch
    stream = torch.cuda.Stream(device)
    fns = [chk.run_append, chk.run_attn]
    for _ in range(args.warmup):
        for f in fns:
            f(stream)
    stream.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    with ClockSampler(local, clocks_dir) as clocks:
        barrier(dist, device)
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        per_fn = timed_loop(args.steps, fns, stream)
        t_end.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        barrier(dist, device)
    step_ms = t_start.elapsed_time(t_end) / args.steps
    app_ms, attn_ms = max_over_ranks(dist, per_fn, device)
    step_ms = max_over_ranks(dist, [step_ms], device)[0]
    return step_ms, app_ms, attn_ms, clocks


def run_chunk(args, chk, dist, rank, world, local, device):
    """Bench line of a chunked-prefill workload (device-timed; no e2e leg)."""
    step_ms, app_ms, attn_ms, clocks = time_chunk(args, chk, dist, local, device,
                                                  args.clocks_log_dir)
    tflops = chk.flops / ((app_ms + attn_ms) * 1e-3) / 1e12 * world
    kern = chk.flops / (attn_ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "gpu_launches": args.steps * chk.launches,
            "roofline": tensor_roofline(kern, "attn_prefill_paged_kernel",
                                        MEASURED_TRAFFIC.get(chk.spec.name), clocks.summary()),
            "chunk": {"sconv_append_ms": app_ms, "attn_prefill_paged_ms": attn_ms},
            "config": {"workload": chk.spec.name, "parallelism": f"replica per GPU x{world}",
                       "l2": chk.l2_note},
            "e2e": None, "clocks": clocks.summary()}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, thr = oracle_chunk_sample(chk.spec, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def run_sconv_out(args, spec, dist, rank, world, local, device):
    """Bench line of the output sconv (HBM-bound; device-timed, no e2e leg)."""
    import torch
    import relative_bias_sliding_b200 as ink
    from relative_bias_sliding_b200.inputs import make_sconv_out
    t = make_sconv_out(spec, device=device)
    y = torch.empty_like(t["x"])
    stream = torch.cuda.Stream(device)
    fn = lambda s=None: ink.sconv_out(t["x"], t["w"], t["state"], out=y, stream=s)
    for _ in range(args.warmup):
        fn(stream)
    stream.synchronize()
    barrier(dist, device)
    with ClockSampler(local, args.clocks_log_dir) as clocks:
        torch.cuda.synchronize()
        ms = timed_loop(args.steps, [fn], stream)[0]
        barrier(dist, device)
    ms = max_over_ranks(dist, [ms], device)[0]
    peaks, peak_src = load_peaks()
    gbs = spec.bytes_moved / (ms * 1e-3) / 1e9
    line = {"metric": METRIC, "value": gbs * world, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "gpu_launches": args.steps,
            "roofline": {"bound": "hbm", "kernel": "sconv_out_kernel", "achieved": gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "peak_source": f"{peak_src} hbm_gbs"},
            "config": {"workload": spec.name, "parallelism": f"replica per GPU x{world}",
                       "l2": "inputs larger than L2 (x and y 512 MiB each)"},
            "e2e": None, "clocks": clocks.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def time_with_clocks(args, fns, dist, local, device, steps=None):
    """Warm up, then time ``steps`` (default --steps) passes over ``fns`` on one
    stream with the clocks sampled; per-callable mean ms (max over ranks), the
    whole-pass ms, and the clock summary."""
    import torch
    steps = steps or args.steps
    stream = torch.cuda.Stream(device)
    for _ in range(args.warmup):
        for f in fns:
            f(stream)
    stream.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    with ClockSampler(local, args.clocks_log_dir) as clocks:
        barrier(dist, device)
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        per_fn = timed_loop(steps, fns, stream)
        t_end.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        barrier(dist, device)
    step_ms = t_start.elapsed_time(t_end) / steps
    per_fn = max_over_ranks(dist, per_fn, device)
    step_ms = max_over_ranks(dist, [step_ms], device)[0]
    return per_fn, step_ms, clocks.summary()


def time_graph(args, fn, dist, local, device, steps):
    """Capture one call of ``fn`` in a CUDA graph, warm up, then time ``steps``
    replays on one stream with the clocks sampled (the way a server runs a
    launch-bound shape).  Returns mean ms per replay (max over ranks) and the
    clock summary."""
    import torch
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(side):
        for _ in range(3):  # first calls outside the capture (attributes, caches)
            fn(side)
    side.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn(torch.cuda.current_stream(device))
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
        stream.synchronize()
        barrier(dist, device)
        with ClockSampler(local, args.clocks_log_dir) as clocks:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                graph.replay()
            b.record(stream)
            stream.synchronize()
        barrier(dist, device)
    ms = max_over_ranks(dist, [a.elapsed_time(b) / steps], device)[0]
    del graph
    return ms, clocks.summary()


def prefill_parts(args, pre, dist, device):
    """(sconv ms, paged-kernel ms) of a two-pass prefill call, its two kernels
    timed apart as the two public calls that launch them on the same layout
    (PrefillStep.add_parts); None on the fused path."""
    if not pre.two_pass:
        return None
    pre.add_parts(device)
    parts = time_loop_only(args, [pre.run_part_sconv, pre.run_part_attn], dist, device)
    del pre.p_kc, pre.p_vc
    return parts


def prefill_roofline(pre, call_ms, parts, clocks):
    """Roofline of the call's dominant kernel (the paged prefill kernel on the
    two-pass path, the fused kernel otherwise) and the path record."""
    kern_ms = parts[1] if parts else call_ms
    key = pre.spec.name + ("" if pre.two_pass else " fused")
    roof = tensor_roofline(pre.flops / (kern_ms * 1e-3) / 1e12, pre.kernel,
                           MEASURED_TRAFFIC.get(key), clocks)
    path = {"path": pre.path, "call_ms": call_ms}
    if parts:
        path.update({"sconv_ms": parts[0], "attn_prefill_paged_ms": parts[1],
                     "kernel_timing": "the call's two kernels timed apart, as the public "
                                      "sconv append and paged prefill on the same block layout"})
    return roof, path


def prefill_object(args, pre, ms, step_ms, steps, world, clocks, with_cpu, dist=None,
                   device=None):
    """Bench sub-object of one prefill workload on the automatic path."""
    tflops = pre.flops / (ms * 1e-3) / 1e12
    parts = prefill_parts(args, pre, dist, device)
    roof, path = prefill_roofline(pre, ms, parts, clocks)
    obj = {"workload": pre.spec.name, "value": tflops * world, "unit": "TFLOP/s",
           "ms_per_step": step_ms, "steps": steps, "gpu_launches": steps * pre.launches,
           "flops_per_step": pre.flops, "prefill_path": path, "roofline": roof,
           "clocks": clocks}
    if with_cpu:
        v, desc, thr = oracle_prefill_sample(pre.spec, args.cpu_seconds)
        obj["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                               "sample": desc}
    return obj


def decode_object(dec, app_ms, attn_ms, step_ms, steps, world, clocks):
    """Bench sub-object of one decode workload: value = key/value bytes per
    step over (sconv append + decode); the roofline is the decode kernels
    alone."""
    gbs = dec.kv_bytes / ((app_ms + attn_ms) * 1e-3) / 1e9
    kern = dec.kv_bytes / (attn_ms * 1e-3) / 1e9
    mq = dec.spec.n_new > 1
    kernel = ("decode_mq_tc_kernel" if mq else "decode_split_kernel") + \
        (" + decode_combine_kernel" if dec.splits > 1 else "")
    return {"workload": dec.spec.name, "value": gbs * world, "unit": "GB/s",
            "ms_per_step": step_ms, "steps": steps, "gpu_launches": steps * dec.launches,
            "sconv_append_ms": app_ms, "attn_decode_ms": attn_ms, "num_splits": dec.splits,
            "kv_bytes_per_step": dec.kv_bytes,
            "roofline": hbm_roofline(kern, kernel, MEASURED_TRAFFIC.get(dec.spec.name)),
            "clocks": clocks}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import relative_bias_sliding_b200 as ink
    from relative_bias_sliding_b200.inputs import WORKLOADS, PrefillSpec, ChunkSpec, SconvOutSpec

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    ink.load_library()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline

    if args.workload:
        spec = WORKLOADS[args.workload]
        if isinstance(spec, SconvOutSpec):
            return run_sconv_out(args, spec, dist, rank, world, local, device)
        if isinstance(spec, ChunkSpec):
            return run_chunk(args, ChunkStep(spec, device), dist, rank, world, local, device)
        pre = PrefillStep(spec, device, args.prefill_path) if isinstance(spec, PrefillSpec) else None
        dec = None if pre else DecodeStep(spec, device)
    else:
        pre = PrefillStep(WORKLOADS[DEFAULT_PREFILL], device, args.prefill_path)
        dec = DecodeStep(WORKLOADS[DEFAULT_DECODE], device)
    fns = []
    if pre:
        fns.append(pre.run)
    if dec:
        fns += [dec.run_append, dec.run_attn]

    per_fn, step_ms, clocks = time_with_clocks(args, fns, dist, local, device)
    stream = torch.cuda.Stream(device)

    e2e = None
    if not args.no_e2e:
        e2e_parts = []
        if pre:
            e2e_parts.append(("pre",) + e2e_prefill(pre, max(10, args.steps), stream))
        if dec:
            e2e_parts.append(("dec",) + e2e_decode(dec, max(10, args.steps), stream))
        e2e = e2e_parts

    line = {"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "gpu_launches": args.steps * sum(x.launches for x in (pre, dec) if x)}
    i = 0
    if pre:
        pre_ms = per_fn[0]
        i = 1
        tflops = pre.flops / (pre_ms * 1e-3) / 1e12 * world
        line.update({"value": tflops, "unit": "TFLOP/s"})
        line["roofline"], line["prefill_path"] = prefill_roofline(
            pre, pre_ms, prefill_parts(args, pre, dist, device), clocks)
    if dec:
        app_ms, attn_ms = per_fn[i], per_fn[i + 1]
        dec_obj = decode_object(dec, app_ms, attn_ms, app_ms + attn_ms, args.steps, world,
                                clocks)
        del dec_obj["clocks"]
        if pre:
            line["decode"] = dec_obj
        else:
            line.update({"value": dec_obj["value"], "unit": "GB/s",
                         "roofline": dec_obj["roofline"]})
            line["decode"] = {k: v for k, v in dec_obj.items() if k != "roofline"}
    sizes = []
    if pre:
        sizes.append(f"prefill q {pre.t['q'].numel() * 2 / 2**20:.0f} MiB")
    if dec:
        sizes.append(f"decode K/V cache {dec.cache_bytes / 1e9:.1f} GB")
    line["config"] = {"workload": (pre.spec.name if pre else "") +
                      (" + " if pre and dec else "") + (dec.spec.name if dec else ""),
                      "parallelism": f"replica per GPU x{world}",
                      "l2": "inputs larger than L2 (" + "; ".join(sizes) + ")"}
    if pre:
        line["config"]["prefill_path"] = args.prefill_path
    if e2e:
        parts = {p[0]: p[1:] for p in e2e}
        if pre:
            ms, h2d, d2h = parts["pre"]
            line["e2e"] = {"value": pre.flops / (ms * 1e-3) / 1e12 * world, "unit": "TFLOP/s",
                           "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                           "steps": max(10, args.steps),
                           "pipelined": "copy-in, compute and copy-out of successive steps "
                                        "overlap on three streams"}
            if dec:
                ms2, h2d2, d2h2 = parts["dec"]
                line["e2e"]["decode"] = {"value": dec.kv_bytes / (ms2 * 1e-3) / 1e9 * world,
                                         "unit": "GB/s", "ms_per_step": ms2,
                                         "h2d_bytes_per_step": h2d2, "d2h_bytes_per_step": d2h2}
        else:
            ms2, h2d2, d2h2 = parts["dec"]
            line["e2e"] = {"value": dec.kv_bytes / (ms2 * 1e-3) / 1e9 * world, "unit": "GB/s",
                           "ms_per_step": ms2, "h2d_bytes_per_step": h2d2,
                           "d2h_bytes_per_step": d2h2}
    line["clocks"] = clocks

    if not args.workload:
        # the same prefill on the fused kernel (sconv applied to each key/value
        # tile on its way to the tensor cores), timed on its own after the step
        fu_ms = time_loop_only(args, [pre.run_fused], dist, device)[0]
        fu = pre.flops / (fu_ms * 1e-3) / 1e12
        line["prefill_fused"] = {
            "workload": pre.spec.name, "value": fu * world, "unit": "TFLOP/s",
            "ms_per_step": fu_ms, "gpu_launches": args.steps,
            "roofline": tensor_roofline(fu, "attn_prefill_pair_kernel",
                                        MEASURED_TRAFFIC.get(pre.spec.name + " fused"), clocks)}
        # the same prefill also writing the paged cache and the sconv state,
        # on the automatic path and on the fused kernel
        pre.add_cache(device)
        f_ms, ff_ms = time_loop_only(args, [pre.run_fill, pre.run_fill_fused], dist, device)
        line["prefill_fills_cache"] = {
            "workload": pre.spec.name, "value": pre.flops / (f_ms * 1e-3) / 1e12 * world,
            "unit": "TFLOP/s", "ms_per_step": f_ms, "path": pre.path,
            "gpu_launches": args.steps * (pre.launches + 1),
            "cache_bytes_written": pre.spec.B * pre.spec.T * pre.spec.Hkv * 128 * 2 * 2,
            "plain_ms_per_step": per_fn[0],
            "fused": {"value": pre.flops / (ff_ms * 1e-3) / 1e12 * world, "unit": "TFLOP/s",
                      "ms_per_step": ff_ms, "plain_ms_per_step": fu_ms}}
        # the same prefill shape through the paged cache (sconv append of all
        # keys/values, then the paged prefill), timed on its own after the step
        via = ChunkStep(WORKLOADS[DEFAULT_VIA_CACHE], device)
        v_step, v_app, v_attn, v_clocks = time_chunk(args, via, dist, local, device, None)
        v_kern = via.flops / (v_attn * 1e-3) / 1e12
        vc = v_clocks.summary()
        line["prefill_via_cache"] = {
            "workload": via.spec.name, "value": via.flops / ((v_app + v_attn) * 1e-3) / 1e12 * world,
            "unit": "TFLOP/s", "ms_per_step": v_step, "sconv_append_ms": v_app,
            "attn_prefill_paged_ms": v_attn, "gpu_launches": args.steps * via.launches,
            "roofline": tensor_roofline(v_kern, "attn_prefill_paged_kernel",
                                        MEASURED_TRAFFIC.get(via.spec.name), vc),
            "clocks": vc}
        del via
        if with_cpu:
            # the oracle on the decode workload of the step
            v, desc, thr = oracle_decode_sample(dec.spec, args.cpu_seconds)
            line["decode"]["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": thr,
                                              "kind": "oracle", "sample": desc}
        del pre, dec
        torch.cuda.empty_cache()
        # the other workloads of the layer, each timed on its own with its
        # roofline and the oracle timed beside it
        for name in EXTRA_PREFILL:
            p2 = PrefillStep(WORKLOADS[name], device, args.prefill_path)
            steps = max(args.steps, 200) if p2.flops < 1e10 else args.steps
            pf, pstep, pclk = time_with_clocks(args, [p2.run], dist, local, device, steps)
            if p2.flops < 1e10:
                # launch-bound: the same call captured in a CUDA graph and
                # replayed (the host-side argument checks and tensor-map
                # encoding leave the replay); the eager figure is kept beside
                gms, gclk = time_graph(args, p2.run, dist, local, device, steps)
                obj = prefill_object(args, p2, gms, gms, steps, world, gclk, with_cpu)
                obj["launch"] = "CUDA graph replay of one captured call"
                obj["eager"] = {"value": p2.flops / (pf[0] * 1e-3) / 1e12 * world,
                                "unit": "TFLOP/s", "ms_per_step": pstep}
                line[name] = obj
            else:
                line[name] = prefill_object(args, p2, pf[0], pstep, steps, world, pclk, with_cpu,
                                            dist, device)
            del p2
            torch.cuda.empty_cache()
        for name in EXTRA_DECODE:
            d2 = DecodeStep(WORKLOADS[name], device)
            df, dstep, dclk = time_with_clocks(args, [d2.run_append, d2.run_attn], dist, local,
                                               device)
            obj = decode_object(d2, df[0], df[1], dstep, args.steps, world, dclk)
            if with_cpu:
                if d2.spec.L_min >= (1 << 16):
                    v, desc, thr = oracle_decode_long_sample(d2)
                else:
                    v, desc, thr = oracle_decode_sample(d2.spec, args.cpu_seconds)
                obj["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": thr,
                                       "kind": "oracle", "sample": desc}
            line[name] = obj
            del d2
            torch.cuda.empty_cache()
        line["gpu_launches_all"] = (line["gpu_launches"] + line["prefill_fused"]["gpu_launches"]
                                    + line["prefill_fills_cache"]["gpu_launches"]
                                    + line["prefill_via_cache"]["gpu_launches"]
                                    + sum(line[n]["gpu_launches"] for n in EXTRA_PREFILL + EXTRA_DECODE))

    if with_cpu:
        if args.workload and pre:
            v, desc, thr = oracle_prefill_sample(pre.spec, args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": thr,
                                    "kind": "oracle", "sample": desc}
        elif args.workload:
            if dec.spec.L_min >= (1 << 16):
                v, desc, thr = oracle_decode_long_sample(dec)
            else:
                v, desc, thr = oracle_decode_sample(dec.spec, args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": thr,
                                    "kind": "oracle", "sample": desc}
        else:
            v, desc, thr = oracle_prefill_sample(WORKLOADS[DEFAULT_PREFILL], args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": thr,
                                    "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
