"""Multi-rank host logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

`bench.py --gpus N` runs one process per GPU: each rank ranks its own prefill sequence (weak scaling,
no collective on the data path), the job's time is the slowest rank's, and the value counts every
rank's pairs.  These are exercised here without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                         world_size=world)
    try:
        import bench
        slowest = bench.max_over_ranks(1.5 * (rank + 1), world)   # rank r's step time
        bench.barrier(world)
        b = bench.rank_workload(rank, T=64)
        q.put((rank, slowest, float(b.Q.float().sum()), b.eligible_pairs(),
               bench.job_value(b.eligible_pairs(), world, slowest)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_own_sequences():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, m0, s0, p0, v0), (_, m1, s1, p1, v1) = out
    assert m0 == m1 == 3.0                      # both ranks see the slowest rank's time
    assert s0 != s1                             # each rank has its own sequence
    assert p0 == p1 == 64 * 65 // 2             # same shape: weak scaling
    assert v0 == v1 == pytest.approx(2 * p0 / 3e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    bench.barrier(1)
