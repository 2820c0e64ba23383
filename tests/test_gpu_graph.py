"""The library's calls captured in a CUDA graph and replayed give the eager
results bit for bit: the prefill, and a decode step (sconv append + decode
with the automatic split plan)."""
import pytest
import torch

from conftest import need_gpu
import relative_bias_sliding_b200 as ink
from relative_bias_sliding_b200.inputs import WORKLOADS, make_decode, make_prefill, scaled

pytestmark = pytest.mark.gpu


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(side)  # first call outside the capture
    side.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn(torch.cuda.current_stream())
    return graph


@pytest.mark.parametrize("name,T", [("prefill_tiny_b1_t256", 256),
                                    ("prefill_swa_b1_t8192", 1000),
                                    ("prefill_swa_b1_t8192", 2500)])
def test_prefill_graph_replay_matches_eager(name, T):
    """256 and 1000 tokens take the fused kernel, 2500 the two-pass path (two
    kernels, with the scratch allocated by the binding during capture)."""
    need_gpu()
    spec = WORKLOADS[name]
    if T != spec.T:
        spec = scaled(spec, T=T)  # several query blocks and a ragged tail
    t = make_prefill(spec, device="cuda")
    args = (t["q"], t["k_raw"], t["v_raw"], t["w_k"], t["w_v"], t["bias"])
    eager = ink.attn_prefill(*args, window=spec.window)
    out = torch.empty_like(eager)
    graph = _capture(lambda s: ink.attn_prefill(*args, window=spec.window, out=out, stream=s))
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)


@pytest.mark.parametrize("S,n_new", [(8, 1), (48, 1), (48, 3)])
def test_decode_step_graph_replay_matches_eager(S, n_new):
    """48 sequences fill the SMs' slots, so the automatic plan runs some of
    them in pieces merged by the combine (two kernels in the graph)."""
    need_gpu()
    spec = scaled(WORKLOADS["decode_swa_s64"], S=S, L_min=500, L_max=5000, n_new=n_new, seed=31)
    t = make_decode(spec, device="cuda")
    keep = {k: t[k].clone() for k in ("k_cache", "v_cache", "k_state", "v_state")}

    def step(out, s=None):
        ink.sconv_kv(t["k_new"], t["v_new"], t["w_k"], t["w_v"], t["k_state"], t["v_state"],
                     t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"], stream=s)
        ink.attn_decode(t["q"], t["k_cache"], t["v_cache"], t["block_table"], t["seq_lens"],
                        t["bias"], window=spec.window, out=out, stream=s)

    def restore():
        for k, v in keep.items():
            t[k].copy_(v)

    eager = torch.empty_like(t["q"])
    step(eager)
    torch.cuda.synchronize()
    after = {k: t[k].clone() for k in keep}
    restore()
    out = torch.empty_like(t["q"])
    graph = _capture(lambda s: step(out, s))
    restore()
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    for k in keep:
        assert torch.equal(t[k], after[k]), k
