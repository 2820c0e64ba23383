"""Host-side bookkeeping of bench.py and of the profiler summaries, on CPU:
the commands under profiles/ run workloads and flags that exist, the DRAM
traffic table names real workloads, and the roofline object of a prefill
step picks the traffic of the kernel its path actually ran."""
import importlib.util
import os
import shlex
import sys

import pytest

from relative_bias_sliding_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _bench_commands():
    """Every `python bench.py ...` command line in the profiler summaries
    (backslash continuations joined)."""
    out = []
    pdir = os.path.join(ROOT, "profiles")
    for name in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, name)).read().replace("\\\n", " ")
        for line in text.splitlines():
            i = line.find("python bench.py")
            if i >= 0:
                out.append((name, line[i + len("python "):].strip()))
    return out


def test_profiles_hold_text_summaries_only():
    pdir = os.path.join(ROOT, "profiles")
    for name in os.listdir(pdir):
        assert name.endswith((".md", ".txt")), name


@pytest.mark.parametrize("name,cmd", _bench_commands())
def test_profile_commands_parse_and_name_existing_workloads(name, cmd, monkeypatch):
    """The bench command each summary gives still parses, and its workload
    exists, so the capture it describes can be repeated."""
    bench = _bench()
    argv = shlex.split(cmd)
    assert argv[0] == "bench.py", (name, cmd)
    monkeypatch.setattr(sys, "argv", argv)
    args = bench.parse()
    if args.workload is not None:
        assert args.workload in WORKLOADS, (name, args.workload)


def test_every_profile_gives_its_command():
    pdir = os.path.join(ROOT, "profiles")
    for name in os.listdir(pdir):
        text = open(os.path.join(pdir, name)).read()
        assert "python bench.py" in text, name
        # every ncu capture keeps the GPU clocks as they are
        for line in text.replace("\\\n", " ").splitlines():
            cmdline = line.strip()
            if cmdline.startswith("ncu ") and ("--metrics" in cmdline or "--set" in cmdline):
                assert "--clock-control none" in cmdline, (name, cmdline)


def test_traffic_table_names_real_workloads():
    bench = _bench()
    for key, nbytes in bench.MEASURED_TRAFFIC.items():
        base = key[:-len(" fused")] if key.endswith(" fused") else key
        assert base in WORKLOADS, key
        assert nbytes > 0


class _Pre:
    def __init__(self, name, two_pass):
        self.spec = WORKLOADS[name]
        self.flops = self.spec.flops
        self.two_pass = two_pass
        self.path = "two_pass" if two_pass else "fused"
        self.kernel = "attn_prefill_paged_kernel" if two_pass else "attn_prefill_pair_kernel"


def test_prefill_roofline_uses_the_traffic_of_the_path_taken():
    bench = _bench()
    name = "prefill_swa_b4_t8192"
    two = _Pre(name, True)
    roof, path = bench.prefill_roofline(two, 4.2, (0.07, 4.1), None)
    assert roof["kernel"] == "attn_prefill_paged_kernel"
    assert roof["traffic"] == bench.MEASURED_TRAFFIC[name]
    assert roof["achieved"] == pytest.approx(two.flops / 4.1e-3 / 1e12)  # the kernel's own time
    assert path["path"] == "two_pass" and path["attn_prefill_paged_ms"] == 4.1
    fused = _Pre(name, False)
    roof, path = bench.prefill_roofline(fused, 4.7, None, None)
    assert roof["kernel"] == "attn_prefill_pair_kernel"
    assert roof["traffic"] == bench.MEASURED_TRAFFIC[name + " fused"]
    assert roof["achieved"] == pytest.approx(fused.flops / 4.7e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    # a workload with no capture of its kernel reports no traffic
    roof, _ = bench.prefill_roofline(_Pre("prefill_tiny_b1_t256", False), 0.02, None, None)
    assert roof["traffic"] is None
