"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

With more than one GPU, bench.py splits the heads of one layer across the
ranks (heads are independent in every step of the path; g, the coverage flags
and the neighbour table are shared inputs), or gives every rank its own layer
(--shard layers).  Neither needs a data-path collective.  What can be checked
without GPUs is the host side: the head partition covers every head exactly
once, a rank's share of the inputs is the matching slice of the single-rank
draw, the per-rank results of the oracle put together are the single-rank
results, and the job throughput is the sum of the ranks' FLOPs over the
slowest rank's step time.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawn(target, world, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q, *args)) for r in range(world)]
    for p in procs:
        p.start()
    # drain the queue before joining: a child holding a large result in the
    # queue cannot exit until it has been read
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    return out


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))


def _aggregate_worker(rank, world, port, q):
    _init(rank, world, port)
    try:
        import bench
        flops = 1e12 * (rank + 1)          # rank 0: 1 TFLOP, rank 1: 2 TFLOP
        ms = 2.0 if rank == 0 else 4.0     # rank 1 is the slowest
        value, ms_max = bench.aggregate(flops, ms, world, device="cpu")
        wl_h, heads = bench.rank_workload(rank, world, shard="heads")
        wl_l, _ = bench.rank_workload(rank, world, shard="layers")
        q.put((rank, value, ms_max, heads, wl_h.layer, wl_l.layer, wl_l.seed))
    finally:
        dist.destroy_process_group()


def test_two_ranks_aggregation_and_shares():
    res = sorted(_spawn(_aggregate_worker, 2))
    (r0, v0, m0, hd0, lh0, ll0, s0), (r1, v1, m1, hd1, lh1, ll1, s1) = res
    assert m0 == m1 == 4.0                                    # max over ranks
    assert abs(v0 - 3e12 / 4e-3 / 1e12) < 1e-9 and v0 == v1   # sum FLOPs / max time
    assert hd0 == (0, 20) and hd1 == (20, 40)                 # one layer, heads split
    assert lh0 == lh1 == 0
    assert (ll0, ll1) == (0, 1) and s0 != s1                  # --shard layers: own layer


@pytest.mark.parametrize("H", [1, 3, 7, 40])
def test_head_ranges_cover_every_head_once(H):
    import bench
    for world in range(1, H + 1):
        ranges = [bench.head_range(r, world, H) for r in range(world)]
        heads = [h for (a, b) in ranges for h in range(a, b)]
        assert heads == list(range(H))                        # each head exactly once, in order
        sizes = [b - a for (a, b) in ranges]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_head_slice_of_inputs_is_the_single_rank_draw():
    from synth import make_inputs
    from synth.configs import small
    wl = small(5, 2, 9, 2)
    full = make_inputs(wl, "cpu")
    for (a, b) in [(0, 2), (2, 5), (4, 5)]:
        part = make_inputs(wl, "cpu", heads=(a, b))
        assert part.wl.heads == b - a
        for name in ("Q", "K", "V"):
            assert torch.equal(getattr(part, name), getattr(full, name)[a:b])
        assert torch.equal(part.g, full.g) and torch.equal(part.covered, full.covered)


def _oracle_layer(inp, heads):
    """Oracle importance -> route -> attention for the given heads of inp."""
    from oracle import attention as oatt
    from oracle import importance as oimp
    from oracle import route as ort
    wl = inp.wl
    prm = ort.Params(lam=wl.params.lam, tau=wl.params.tau, g_ref=wl.params.g_ref,
                     theta_cov=wl.params.theta_cov, theta_unc=wl.params.theta_unc,
                     k_cov=wl.params.k_cov, k_unc=wl.params.k_unc)
    g, cov = inp.g.numpy(), inp.covered.numpy()
    out = []
    for h in heads:
        Q, K, V = (x[h].to(torch.float64).numpy() for x in (inp.Q, inp.K, inp.V))
        p = oimp.importance(Q, K, wl.b, 1.0).astype(np.float32)
        for i in range(wl.n_q_blocks):
            bud, ext, _ = ort.route_row(p[i], g[i], bool(cov[i]), prm, wl.prev_begin,
                                        wl.prev_count)
            O, lse = oatt.routed_attention_block(Q[i * wl.b:(i + 1) * wl.b], K, V, bud + ext,
                                                 wl.b)
            out.append((bud + ext, O, lse))
    return out


def _layer_worker(rank, world, port, q, H):
    _init(rank, world, port)
    try:
        import bench
        from synth import make_inputs
        from synth.configs import small
        wl = small(H, 2, 9, 2)
        a, b = bench.head_range(rank, world, H)
        part = make_inputs(wl, "cpu", heads=(a, b))
        mine = _oracle_layer(part, range(b - a))
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        q.put((rank, gathered))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_shares_concatenate_to_the_single_rank_layer():
    from synth import make_inputs
    from synth.configs import small
    H = 3  # not divisible by the world size
    res = dict(_spawn(_layer_worker, 2, H))
    joined = res[0][0] + res[0][1]
    assert res[1][0] is not None
    whole = _oracle_layer(make_inputs(small(H, 2, 9, 2), "cpu"), range(H))
    assert len(joined) == len(whole)
    for (ids_a, O_a, l_a), (ids_b, O_b, l_b) in zip(joined, whole):
        assert ids_a == ids_b
        assert np.array_equal(O_a, O_b) and np.array_equal(l_a, l_b)


def test_single_rank_aggregation_is_identity():
    import bench
    v, ms = bench.aggregate(2e12, 4.0, 1, device="cpu")
    assert ms == 4.0 and abs(v - 500.0) < 1e-9
