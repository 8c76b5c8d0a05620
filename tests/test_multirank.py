"""The multi-GPU mode is replicas only: every rank runs its own copy of the
workload and bench.py only needs a barrier and a max over ranks.  These run
as two gloo processes on CPU, plus checks of the algorithmic work counts."""
import os
import socket

import numpy as np
import pytest

import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank), PA_BENCH_BACKEND="gloo")
    import torch.distributed as dist

    import bench
    r, w, _ = bench.dist_setup(world)
    v = bench.max_over_ranks(10.0 * (r + 1), w)
    bench.barrier(w)
    q.put((r, w, v))
    dist.destroy_process_group()


def test_two_rank_max_and_barrier_over_gloo():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, 2, 20.0), (1, 2, 20.0)]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_algorithmic_counts_by_hand():
    import bench
    spec = workloads.custom([1, 3], [4, 0], 4, 2, 8, 4)
    c = bench.algorithmic_counts(spec)
    # T = 5 and 3; K/V bytes = sum T * kvh * d * 2 (f16) * 2 (K and V).
    assert c["kv_bytes"] == (5 + 3) * 2 * 8 * 4
    assert c["q_bytes"] == 4 * 4 * 8 * 2
    # visible pairs: seq0 row 0 sees 5 keys; seq1 rows see 1, 2, 3 keys.
    assert c["flops"] == 4 * 4 * 8 * (5 + 1 + 2 + 3)
    assert c["scatter_bytes"] == 4 * 4 * 2 * 8 * 2 + 4 * 4
    assert c["decode"] is True
