"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): ranks run
independent replicas, timings are reduced with max over ranks, and only rank 0
reports.  No data-path collective exists on the layer's path."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    # rank-dependent "times": the reduction must return the slowest rank's
    vals = bench.max_over_ranks(dist, [1.0 + rank, 5.0 - rank, float(rank)])
    bench.barrier(dist)
    # the reference arm does no work on ranks other than 0
    class A:
        workload = "prefill_tiny_b1_t256"
        steps, warmup, gpus = 1, 0, world
    rc = bench.run_reference(A) if rank != 0 else 0
    dist.destroy_process_group()
    q.put((rank, vals, rc))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, vals, rc in out:
        assert vals == [2.0, 5.0, 1.0]
        assert rc == 0


def test_single_rank_has_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(None, [3.0, 1.0]) == [3.0, 1.0]


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def _oracle_sconv_inplace(xs, w_shard, state_shard):
    """The oracle's sconv standing in, on the CPU, for the library's kernel in
    the channel-sharded output sconv (test infrastructure: only the collective
    logic around it is under test here).  Updates state_shard in place."""
    import numpy as np
    import torch
    import oracle
    y = oracle.sconv(_bits(xs), w_shard.numpy(), None if state_shard is None else _bits(state_shard))
    if state_shard is not None:
        hist = torch.cat([state_shard, xs], dim=1)
        state_shard.copy_(hist[:, -3:])
    return torch.from_numpy(np.ascontiguousarray(y).view(np.int16)).view(torch.bfloat16)


def _sconv_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from relative_bias_sliding_b200.sharded import channel_shard, sconv_out_reduce_scatter
    dist.init_process_group("gloo", rank=rank, world_size=world)
    B, T, C = 2, 70, 64
    g = torch.Generator().manual_seed(100)  # the same draws on every rank
    xs = [torch.randn(B, T, C, generator=g).to(torch.bfloat16) for _ in range(world)]
    w = torch.randn(C, 4, generator=g) * 0.5
    state = torch.randn(B, 3, C, generator=g).to(torch.bfloat16)
    sl = channel_shard(C, world, rank)
    st = state[:, :, sl].clone()
    y = sconv_out_reduce_scatter(xs[rank], w, st, local_sconv=_oracle_sconv_inplace)
    y2 = sconv_out_reduce_scatter(xs[rank], w, st, local_sconv=_oracle_sconv_inplace)
    dist.destroy_process_group()
    q.put((rank, _bits(y).copy(), _bits(y2).copy(), _bits(st).copy()))


def test_channel_sharded_output_sconv_gloo_world2():
    """Two ranks each hold a partial sum of the output sconv's input; the
    reduce-scatter / sconv-of-the-shard / all-gather path returns on every
    rank the unsharded sconv of the summed input, bit for bit, twice in a row
    (the second call continues from the state shards), and each rank's state
    shard equals its slice of the unsharded state."""
    import torch
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_sconv_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {r: (y, y2, st) for r, y, y2, st in (q.get(timeout=120) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # unsharded reference on one process: sum in fp32, one bf16 rounding,
    # sconv of all channels from the full state, twice
    sys.path.insert(0, ROOT)
    from relative_bias_sliding_b200.sharded import channel_shard
    B, T, C = 2, 70, 64
    g = torch.Generator().manual_seed(100)
    xs = [torch.randn(B, T, C, generator=g).to(torch.bfloat16) for _ in range(world)]
    w = torch.randn(C, 4, generator=g) * 0.5
    state = torch.randn(B, 3, C, generator=g).to(torch.bfloat16)
    s = (xs[0].float() + xs[1].float()).to(torch.bfloat16)
    y_ref = _oracle_sconv_inplace(s, w, state)
    y2_ref = _oracle_sconv_inplace(s, w, state)
    for r in range(world):
        y, y2, st = out[r]
        assert (y == _bits(y_ref)).all(), f"rank {r}: first call"
        assert (y2 == _bits(y2_ref)).all(), f"rank {r}: second call"
        assert (st == _bits(state[:, :, channel_shard(C, world, r)])).all(), f"rank {r}: state"


def test_shard_selection_covers_every_head_and_channel_once():
    """kv_head_shard / channel_shard: the ranks' slices tile the heads and the
    channels exactly once, in order, and each rank's query heads are the ones
    that read its kv heads (contiguous grouping h -> h / (Hq / Hkv))."""
    sys.path.insert(0, ROOT)
    from relative_bias_sliding_b200.sharded import channel_shard, kv_head_shard
    for Hq, Hkv, world in [(64, 8, 1), (64, 8, 2), (64, 8, 4), (64, 8, 8), (16, 4, 2), (6, 2, 2)]:
        G = Hq // Hkv
        qs, ks, cs = [], [], []
        for r in range(world):
            q, k, c = kv_head_shard(Hq, Hkv, world, r)
            qs += list(range(Hq))[q]
            ks += list(range(Hkv))[k]
            cs += list(range(Hkv * 128))[c]
            assert all(h // G in list(range(Hkv))[k] for h in list(range(Hq))[q])
        assert qs == list(range(Hq)) and ks == list(range(Hkv)) and cs == list(range(Hkv * 128))
    for C, world in [(1024, 1), (1024, 2), (8192, 8)]:
        got = []
        for r in range(world):
            got += list(range(C))[channel_shard(C, world, r)]
        assert got == list(range(C))
    with pytest.raises(ValueError):
        kv_head_shard(64, 8, 3, 0)       # 8 kv heads over 3 ranks
    with pytest.raises(ValueError):
        channel_shard(1000, 2, 0)        # channels not a multiple of 8 * ranks
