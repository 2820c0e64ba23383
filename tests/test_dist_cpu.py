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
