"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The routed path has no exchange step, so several GPUs run independent
layers (weak scaling).  What remains to check without GPUs is the host side:
each rank gets its own layer and seeds, and the job throughput is the sum of
the ranks' FLOPs over the slowest rank's step time.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        wl = bench.rank_workload(rank)
        flops = 1e12 * (rank + 1)          # rank 0: 1 TFLOP, rank 1: 2 TFLOP
        ms = 2.0 if rank == 0 else 4.0     # rank 1 is the slowest
        value, ms_max = bench.aggregate(flops, ms, world, device="cpu")
        q.put((rank, wl.layer, wl.seed, value, ms_max))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, l0, s0, v0, m0), (r1, l1, s1, v1, m1) = res
    assert (l0, l1) == (0, 1) and s0 != s1            # own layer, own seeds
    assert m0 == m1 == 4.0                              # max over ranks
    assert abs(v0 - 3e12 / 4e-3 / 1e12) < 1e-9 and v0 == v1   # sum FLOPs / max time


def test_single_rank_aggregation_is_identity():
    import bench
    v, ms = bench.aggregate(2e12, 4.0, 1, device="cpu")
    assert ms == 4.0 and abs(v - 500.0) < 1e-9
