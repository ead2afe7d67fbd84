"""GPU routed / dense attention vs the fp64 oracle.

Routes here come from the oracle (or are written directly), never from the
GPU path.  Sizes span several KV tiles and ragged route lengths; the chunk-48
case runs at full size in the launch configuration the bench times, checked
on sampled (head, query block) rows.
"""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from synth import config, make_inputs
from synth.configs import small
from parity import (assert_attention_close, attention_rows, oracle_importance, oracle_params,
                    oracle_routes)

pytestmark = pytest.mark.gpu


def _routes_tensor(routes, H, N, R_max):
    ids = torch.full((H, N, R_max), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    for (h, i), lst in routes.items():
        ids[h, i, :len(lst)] = torch.tensor(lst, dtype=torch.int32)
        ln[h, i] = len(lst)
    return ids.cuda(), ln.cuda()


def _attend(inp, rid, rlen, R_max, scale=0.0):
    wl = inp.wl
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    O = torch.full((H, N * 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, N * 128), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_block_sparse_attn(inp.Q, inp.K, inp.V, rid, rlen, R_max, H, N, M, 128, 128, scale,
                                O, lse, st)
    torch.cuda.synchronize()
    return O, lse, int(st.item())


def _oracle_route_lists(inp, heads):
    wl = inp.wl
    p = oracle_importance(inp.Q, inp.K, heads)
    p32 = {h: v.astype(np.float32) for h, v in p.items()}
    rr = oracle_routes(p32, inp.g.cpu().numpy(), inp.covered.cpu().numpy(),
                       oracle_params(wl.params), wl.prev_begin, wl.prev_count)
    return {k: v[0] + v[1] for k, v in rr.items()}


@pytest.mark.parametrize("cfg", [1, 2])
def test_attention_configs_oracle_routes(lib, cfg):
    inp = make_inputs(config(cfg), "cuda")
    wl = inp.wl
    H, N = wl.heads, wl.n_q_blocks
    routes = _oracle_route_lists(inp, range(H))
    R_max = max(len(v) for v in routes.values())
    rid, rlen = _routes_tensor(routes, H, N, R_max)
    O, lse, st = _attend(inp, rid, rlen, R_max)
    assert st == 0
    rows = sorted(routes) if cfg == 1 else sorted(routes)[::5]
    ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)


@pytest.mark.slow
def test_attention_chunk48_sampled_rows(lib):
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    rng = np.random.default_rng(0)
    # oracle routes on a few heads; the others get random routes of the same
    # lengths so that the launch is the full-size one
    heads = [0, 21, 39]
    routes = _oracle_route_lists(inp, heads)
    for h in range(H):
        if h in heads:
            continue
        for i in range(N):
            L = 80 if (h + i) % 2 else 150
            extra = rng.choice(M - 48, size=L - 48, replace=False)
            routes[(h, i)] = sorted(set(range(M - 48, M)) | set(int(x) for x in extra))
    R_max = 214
    rid, rlen = _routes_tensor(routes, H, N, R_max)
    O, lse, st = _attend(inp, rid, rlen, R_max)
    assert st == 0
    rows = [(0, 0), (0, 47), (21, 13), (39, 46), (5, 3), (30, 30), (12, 0), (39, 1)]
    ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)
    assert torch.isfinite(O.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("M", [1, 3, 64])
def test_dense_mode(lib, M):
    inp = make_inputs(small(2, 3, M, 0), "cuda")
    O, lse, st = _attend(inp, None, None, 0)
    assert st == 0
    rows = [(h, i) for h in range(2) for i in range(3)]
    ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: range(M))
    assert_attention_close(O, lse, ref)


def test_dense_mode_sweep_shape_sampled(lib):
    wl = small(40, 48, 256, 48)
    inp = make_inputs(wl, "cuda")
    O, lse, st = _attend(inp, None, None, 0)
    rows = [(0, 0), (17, 40), (39, 47)]
    ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: range(256))
    assert_attention_close(O, lse, ref)


def test_ragged_and_edge_routes(lib):
    H, N, M = 2, 5, 37
    inp = make_inputs(small(H, N, M, 0), "cuda")
    routes = {
        (0, 0): [5],                      # single tile
        (0, 1): [],                       # empty route -> zeros, -inf
        (0, 2): list(range(M)),           # full route == dense
        (0, 3): [36, 0, 17, 2],           # unsorted
        (0, 4): [1, 2, 3],
        (1, 0): [33, 34, 35, 36],
        (1, 1): list(range(0, M, 2)),
        (1, 2): [0],
        (1, 3): [7, 8],
        (1, 4): list(range(M - 1, -1, -1)),
    }
    R_max = M
    rid, rlen = _routes_tensor(routes, H, N, R_max)
    O, lse, st = _attend(inp, rid, rlen, R_max)
    assert st == 0
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(routes), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)
    assert torch.all(O[0, 128:256].float() == 0)
    assert torch.all(torch.isneginf(lse[0, 128:256]))


def test_invalid_and_repeated_ids_are_skipped_and_flagged(lib):
    H, N, M = 1, 4, 12
    inp = make_inputs(small(H, N, M, 0), "cuda")
    R_max = 8
    ids = torch.full((H, N, R_max), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    ids[0, 0, :5] = torch.tensor([3, -1, 12, 4, 1000000])   # two bad ids
    ln[0, 0] = 5
    ids[0, 1, :4] = torch.tensor([2, 9, 2, 9])               # repeats
    ln[0, 1] = 4
    ln[0, 2] = 9                                              # > R_max
    ids[0, 3, :2] = torch.tensor([11, 0])
    ln[0, 3] = 2
    O, lse, st = _attend(inp, ids.cuda(), ln.cuda(), R_max)
    assert st & rbs.DEV_BAD_ROUTE_ID and st & rbs.DEV_DUP_ROUTE_ID and st & rbs.DEV_ROUTE_LEN
    want = {(0, 0): [3, 4], (0, 1): [2, 9], (0, 2): [], (0, 3): [11, 0]}
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(want), lambda h, i: want[(h, i)])
    assert_attention_close(O, lse, ref)


def test_softmax_scale_argument(lib):
    H, N, M = 1, 2, 6
    inp = make_inputs(small(H, N, M, 0), "cuda")
    routes = {(0, 0): [0, 2, 5], (0, 1): [1, 4]}
    rid, rlen = _routes_tensor(routes, H, N, 3)
    O, lse, st = _attend(inp, rid, rlen, 3, scale=0.02)
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(routes), lambda h, i: routes[(h, i)],
                         scale=0.02)
    assert_attention_close(O, lse, ref)


def test_large_logits_stay_finite(lib):
    # keys with a strong shared direction: logits of hundreds, a steady
    # stream of new row maxima across tiles (the rescale path)
    H, N, M = 1, 2, 20
    wl = small(H, N, M, 0, key_mean_sigma=3.0)
    inp = make_inputs(wl, "cuda")
    inp.Q.mul_(4.0)
    routes = {(0, 0): list(range(M)), (0, 1): list(range(M - 1, -1, -1))}
    rid, rlen = _routes_tensor(routes, H, N, M)
    O, lse, st = _attend(inp, rid, rlen, M)
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(routes), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)


def test_longest_route_the_abi_allows(lib):
    # R_max = VELOX_MAX_ROUTE (4096): row 0 visits all 4096 tiles (= dense),
    # row 1 a ragged random 1500, row 2 a single tile
    H, N, M = 1, 3, 4096
    wl = small(H, N, M, 0)
    inp = make_inputs(wl, "cuda")
    r = np.random.default_rng(17)
    routes = {(0, 0): list(range(M)),
              (0, 1): sorted(r.choice(M, size=1500, replace=False).tolist()),
              (0, 2): [int(r.integers(M))]}
    R_max = 4096
    rid, rlen = _routes_tensor(routes, H, N, R_max)
    O, lse, st = _attend(inp, rid, rlen, R_max)
    assert st == 0
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(routes), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)


@pytest.mark.slow
def test_routes_at_the_largest_cache_the_abi_allows(lib):
    # M = VELOX_MAX_BLOCKS = 65536 history blocks (2 GB each of K and V for one
    # head): the compaction bitmap is full, tile coordinates reach
    # 65535 * 128.  The oracle sees only the tiles a row lists (attention over
    # the listed tiles is the whole computation), gathered on the device.
    H, N, M = 1, 3, 65536
    inp = make_inputs(small(H, N, M, 0), "cuda")
    routes = {(0, 0): [0, 1, 32768, 65534, 65535],
              (0, 1): [65535],
              (0, 2): list(range(65536 - 300, 65536, 3))}
    R_max = 128
    rid, rlen = _routes_tensor(routes, H, N, R_max)
    O, lse, st = _attend(inp, rid, rlen, R_max)
    assert st == 0
    for (h, i), tiles in routes.items():
        idx = torch.cat([torch.arange(t * 128, (t + 1) * 128) for t in tiles]).cuda()
        Ks, Vs = inp.K[h:h + 1, idx], inp.V[h:h + 1, idx]
        Qs = inp.Q[h:h + 1, i * 128:(i + 1) * 128]
        ref = attention_rows(Qs, Ks, Vs, [(0, 0)], lambda _h, _i: range(len(tiles)))
        assert_attention_close(O[h:h + 1, i * 128:(i + 1) * 128], lse[h:h + 1, i * 128:(i + 1) * 128],
                               ref)
