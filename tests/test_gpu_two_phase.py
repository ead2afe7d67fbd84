"""Two-phase attention (routed history tiles + the current chunk) vs the oracle."""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from oracle import attention as oatt
from synth import config, make_current, make_inputs
from synth.configs import small
from parity import assert_attention_close, f64

pytestmark = pytest.mark.gpu


def _routes(H, N, M, R, seed, min_len=0):
    r = np.random.default_rng(seed)
    ids = torch.full((H, N, R), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    routes = {}
    for h in range(H):
        for i in range(N):
            k = int(r.integers(min_len, R + 1))
            sel = r.choice(M, size=k, replace=False).astype(np.int32)
            ids[h, i, :k] = torch.from_numpy(sel)
            ln[h, i] = k
            routes[(h, i)] = sel.tolist()
    return ids.cuda(), ln.cuda(), routes


def _run(inp, Kc, Vc, rid, rln, R, order=None):
    wl = inp.wl
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    O = torch.full((H, N * 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((H, N * 128), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_two_phase_attn(inp.Q, inp.K, inp.V, rid, rln, R, Kc, Vc, Kc.shape[1] // 128, H, N,
                             M, 128, 128, 0.0, O, lse, st, row_order=order)
    torch.cuda.synchronize()
    return O, lse, int(st.item())


def _oracle(inp, Kc, Vc, rows, tiles_of):
    out = {}
    for (h, i) in rows:
        q = f64(inp.Q[h, i * 128:(i + 1) * 128])
        out[(h, i)] = oatt.two_phase_attention_block(q, f64(inp.K[h]), f64(inp.V[h]), tiles_of(h, i),
                                                     f64(Kc[h]), f64(Vc[h]), 128)
    return out


@pytest.mark.parametrize("H,N,M,R", [(2, 3, 20, 9), (1, 5, 7, 7), (3, 2, 33, 12)])
def test_two_phase_small(lib, H, N, M, R):
    wl = small(H, N, M, 0)
    inp = make_inputs(wl, "cuda")
    Kc, Vc = make_current(wl, "cuda")
    rid, rln, routes = _routes(H, N, M, R, H * 100 + N)
    O, lse, st = _run(inp, Kc, Vc, rid, rln, R)
    assert st == 0
    ref = _oracle(inp, Kc, Vc, sorted(routes), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)


def test_two_phase_dense_history_and_empty_routes(lib):
    H, N, M = 2, 3, 6
    wl = small(H, N, M, 0)
    inp = make_inputs(wl, "cuda")
    Kc, Vc = make_current(wl, "cuda")
    O, lse, st = _run(inp, Kc, Vc, None, None, 0)
    rows = [(h, i) for h in range(H) for i in range(N)]
    assert_attention_close(O, lse, _oracle(inp, Kc, Vc, rows, lambda h, i: range(M)))
    rid = torch.full((H, N, 4), -1, dtype=torch.int32, device="cuda")
    rln = torch.zeros(H, N, dtype=torch.int32, device="cuda")
    O, lse, st = _run(inp, Kc, Vc, rid, rln, 4)
    assert st == 0
    assert_attention_close(O, lse, _oracle(inp, Kc, Vc, rows, lambda h, i: []))


@pytest.mark.slow
def test_two_phase_chunk48_sampled_rows(lib):
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    Kc, Vc = make_current(wl, "cuda")
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    r = np.random.default_rng(3)
    R = 214
    ids = torch.full((H, N, R), -1, dtype=torch.int32)
    ln = torch.zeros(H, N, dtype=torch.int32)
    routes = {}
    for h in range(H):
        for i in range(N):
            L = 80 if (h + i) % 2 else 150
            extra = r.choice(M - 48, size=L - 48, replace=False)
            lst = sorted(set(range(M - 48, M)) | set(int(x) for x in extra))
            ids[h, i, :len(lst)] = torch.tensor(lst, dtype=torch.int32)
            ln[h, i] = len(lst)
            routes[(h, i)] = lst
    rid, rln = ids.cuda(), ln.cuda()
    order = torch.empty(H * N, dtype=torch.int32, device="cuda")
    rbs.velox_route_schedule(rln, H * N, R, order)
    O, lse, st = _run(inp, Kc, Vc, rid, rln, R, order)
    assert st == 0
    rows = [(0, 0), (17, 31), (39, 47), (8, 5)]
    assert_attention_close(O, lse, _oracle(inp, Kc, Vc, rows, lambda h, i: routes[(h, i)]))


@pytest.mark.parametrize("seed", range(8))
def test_two_phase_random_cases(lib, seed):
    # N_cur independent of N, random route lengths (empty ones included),
    # the longest-first row order
    r = np.random.default_rng(3000 + seed)
    H, N, M = int(r.integers(1, 4)), int(r.integers(1, 6)), int(r.integers(1, 40))
    n_cur = int(r.integers(1, 7))
    wl = small(H, N, M, 0, layer=seed)
    inp = make_inputs(wl, "cuda")
    Kc, Vc = make_current(wl, "cuda", n_blocks=n_cur)
    R = int(r.integers(1, M + 1))
    rid, rln, routes = _routes(H, N, M, R, 3100 + seed)
    order = torch.empty(H * N, dtype=torch.int32, device="cuda")
    rbs.velox_route_schedule(rln, H * N, R, order)
    O, lse, st = _run(inp, Kc, Vc, rid, rln, R, order)
    assert st == 0
    ref = _oracle(inp, Kc, Vc, sorted(routes), lambda h, i: routes[(h, i)])
    assert_attention_close(O, lse, ref)
