"""Seeded random shapes and parameters: route build and attention against the
oracle (route ids bit-exact, attention within tolerance), many small cases in
one pass each.  Every case is fixed by its seed."""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from synth import make_inputs
from synth.configs import small
from parity import assert_attention_close, attention_rows

from test_gpu_route import _run_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed", range(12))
def test_route_random_cases(lib, seed):
    r = np.random.default_rng(1000 + seed)
    H, N, M = int(r.integers(1, 4)), int(r.integers(1, 7)), int(r.integers(1, 300))
    x = r.standard_normal((H, N, M)) * r.uniform(0.1, 4.0)
    # some rows with exact ties (a few distinct values)
    if seed % 3 == 0:
        x = np.round(x)
    p = np.exp(x - x.max(-1, keepdims=True))
    p = (p / p.sum(-1, keepdims=True)).astype(np.float32)
    g = np.where(r.random((N, M)) < r.uniform(0, 0.6), r.random((N, M)), 0.0).astype(np.float32)
    cov = (r.random(N) < 0.5).astype(np.uint8)
    prev = int(r.integers(0, min(M, 60) + 1))
    k_cov, k_unc = int(r.integers(0, M + 5)), int(r.integers(0, M + 5))
    prm = rbs.route_params(float(r.choice([0.0, 0.5, 2.0, 5.0])), float(r.uniform(0, 0.5)),
                           float(r.uniform(0.05, 1.0)), float(r.choice([0.3, 0.9, 1.5])),
                           float(r.choice([0.5, 0.9, 0.99])), k_cov, k_unc)
    nbr = [sorted(r.choice(M, size=int(r.integers(0, min(M, 8) + 1)), replace=False).tolist())
           for _ in range(N)]
    ref = sorted(r.choice(M, size=int(r.integers(0, min(M, 3) + 1)), replace=False).tolist())
    _run_case(p, g, cov, prm, M - prev, prev, nbr, ref)


@pytest.mark.parametrize("seed", range(10))
def test_attention_random_cases(lib, seed):
    r = np.random.default_rng(2000 + seed)
    H, N, M = int(r.integers(1, 4)), int(r.integers(1, 6)), int(r.integers(1, 40))
    inp = make_inputs(small(H, N, M, 0, layer=seed), "cuda")
    R_max = int(r.integers(1, M + 1))
    ids = torch.full((H, N, R_max), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    routes = {}
    for h in range(H):
        for i in range(N):
            k = int(r.integers(0, R_max + 1))
            sel = r.choice(M, size=k, replace=False).tolist()
            ids[h, i, :k] = torch.tensor(sel, dtype=torch.int32)
            ln[h, i] = k
            routes[(h, i)] = sel
    scale = float(r.choice([0.0, 0.05, 0.2]))
    O = torch.full((H, N * 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, N * 128), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    order = torch.empty(H * N, dtype=torch.int32, device="cuda")
    rid, rln = ids.cuda(), ln.cuda()
    rbs.velox_route_schedule(rln, H * N, R_max, order)
    rbs.velox_block_sparse_attn(inp.Q, inp.K, inp.V, rid, rln, R_max, H, N, M, 128, 128, scale,
                                O, lse, st, row_order=order)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(routes), lambda h, i: routes[(h, i)],
                         scale)
    assert_attention_close(O, lse, ref)


@pytest.mark.parametrize("seed", range(4))
def test_attention_random_medium_cases(lib, seed):
    # hundreds to thousands of history blocks, routes of up to 300 tiles,
    # up to 2 heads x 24 query blocks; 6 sampled rows per case
    r = np.random.default_rng(4000 + seed)
    H, N, M = int(r.integers(1, 3)), int(r.integers(4, 25)), int(r.integers(100, 3001))
    inp = make_inputs(small(H, N, M, 0, layer=seed), "cuda")
    R_max = int(r.integers(1, min(M, 300) + 1))
    ids = torch.full((H, N, R_max), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    routes = {}
    for h in range(H):
        for i in range(N):
            k = int(r.integers(0, R_max + 1))
            sel = r.choice(M, size=k, replace=False).tolist()
            ids[h, i, :k] = torch.tensor(sel, dtype=torch.int32)
            ln[h, i] = k
            routes[(h, i)] = sel
    O = torch.full((H, N * 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, N * 128), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    order = torch.empty(H * N, dtype=torch.int32, device="cuda")
    rid, rln = ids.cuda(), ln.cuda()
    rbs.velox_route_schedule(rln, H * N, R_max, order)
    rbs.velox_block_sparse_attn(inp.Q, inp.K, inp.V, rid, rln, R_max, H, N, M, 128, 128, 0.0,
                                O, lse, st, row_order=order)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = sorted(routes)
    pick = [rows[int(x)] for x in r.choice(len(rows), size=min(6, len(rows)), replace=False)]
    ref = attention_rows(inp.Q, inp.K, inp.V, sorted(pick), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)
