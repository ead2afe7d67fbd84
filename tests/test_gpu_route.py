"""GPU route build vs the oracle: same fp32 p in, route ids bit-exact."""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from oracle import gilbert
from oracle import route as ort
from synth import config, make_inputs
from synth.configs import small
from parity import check_route_row, gpu_row, oracle_importance, oracle_params, oracle_routes

pytestmark = pytest.mark.gpu


def _run_case(p32, g, covered, prm, prev_begin, prev_count, nbr=None, ref=(), S_max=0):
    """p32: [H][N][M] float32 numpy; returns (#exact, #cut) after checking."""
    H, N, M = p32.shape
    dev = "cuda"
    p = torch.from_numpy(p32).to(dev)
    gt = torch.from_numpy(np.ascontiguousarray(g, dtype=np.float32)).to(dev)
    cv = torch.from_numpy(np.ascontiguousarray(covered, dtype=np.uint8)).to(dev)
    if nbr is not None:
        S_max = max(S_max, max([len(x) for x in nbr] + [1]))
        ids = torch.full((N, S_max), -1, dtype=torch.int32)
        cnt = torch.zeros(N, dtype=torch.int32)
        for i, lst in enumerate(nbr):
            ids[i, :len(lst)] = torch.tensor(lst, dtype=torch.int32)
            cnt[i] = len(lst)
        nbr_ids, nbr_cnt = ids.to(dev), cnt.to(dev)
    else:
        nbr_ids = nbr_cnt = None
        S_max = 0
    ref_t = torch.tensor(list(ref), dtype=torch.int32, device=dev) if len(ref) else None
    kmax = max(prm.k_cov, prm.k_unc, prev_count)
    R_max = max(1, min(M, kmax + S_max + len(ref)))
    rid = torch.full((H, N, R_max), -7, dtype=torch.int32, device=dev)
    rlen = torch.full((H, N), -7, dtype=torch.int32, device=dev)
    rnb = torch.full((H, N), -7, dtype=torch.int32, device=dev)
    ws_bytes = rbs.velox_workspace_size(H, N, M)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rbs.velox_route_build(p, gt, cv, prm, prev_begin, prev_count, nbr_ids, nbr_cnt, S_max,
                          ref_t, len(ref), H, N, M, rid, rlen, rnb, R_max, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    oprm = oracle_params(prm)
    ref_routes = oracle_routes({h: p32[h] for h in range(H)}, g, covered, oprm, prev_begin,
                               prev_count, nbr, ref)
    rid, rlen, rnb = rid.cpu(), rlen.cpu(), rnb.cpu()
    kinds = {"exact": 0, "cut": 0}
    for (h, i), r in ref_routes.items():
        kinds[check_route_row(gpu_row(rid, rlen, rnb, h, i), r, f"row {(h, i)}")] += 1
    return kinds


def _p_from_oracle(inp, scale=1.0):
    wl = inp.wl
    ref = oracle_importance(inp.Q, inp.K, range(wl.heads), scale)
    return np.stack([ref[h] for h in range(wl.heads)]).astype(np.float32)


def _prm(wl, **kw):
    p = wl.params
    d = dict(lam=p.lam, tau=p.tau, g_ref=p.g_ref, theta_cov=p.theta_cov, theta_unc=p.theta_unc,
             k_cov=p.k_cov, k_unc=p.k_unc)
    d.update(kw)
    return rbs.route_params(**d)


@pytest.mark.parametrize("cfg", [1, 2])
def test_route_configs(lib, cfg):
    inp = make_inputs(config(cfg), "cpu")
    wl = inp.wl
    p32 = _p_from_oracle(inp)
    kinds = _run_case(p32, inp.g.numpy(), inp.covered.numpy(), _prm(wl), wl.prev_begin,
                      wl.prev_count)
    assert kinds["exact"] >= wl.heads * wl.n_q_blocks - 1


@pytest.mark.slow
def test_route_chunk48(lib):
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    p32 = _p_from_oracle(inp)
    T, Hl, Wl = wl.lattice
    nbr = gilbert.neighbour_blocks(T, Hl, Wl, wl.n_chunks, 128, wl.q_chunk,
                                   wl.cache_first_block, wl.n_kv_blocks)
    kinds = _run_case(p32, inp.g.cpu().numpy(), inp.covered.cpu().numpy(), _prm(wl),
                      wl.prev_begin, wl.prev_count, nbr=nbr)
    assert kinds["cut"] <= 2


@pytest.mark.slow
def test_route_chunk48_live_safeguards(lib):
    """The chunk-48 layer with only the last 6 blocks reserved: the 26-
    neighbour blocks of the query blocks in the chunk's first frame (blocks
    2244-2255, the last frame of the previous chunk) are then mostly outside
    the reserved set, so the safeguard append is live.  All 40 heads, GPU p
    fed to both sides; route ids bit-exact."""
    from routed_block_sparse_b200.pipeline import layer_for
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    p32 = layer.importance(inp.Q, inp.K).cpu().numpy()
    T, Hl, Wl = wl.lattice
    M = wl.n_kv_blocks
    nbr = gilbert.neighbour_blocks(T, Hl, Wl, wl.n_chunks, 128, wl.q_chunk,
                                   wl.cache_first_block, M)
    g, cov = inp.g.cpu().numpy(), inp.covered.cpu().numpy()
    kinds = _run_case(p32, g, cov, _prm(wl), M - 6, 6, nbr=nbr)
    assert kinds["cut"] <= 2
    # the extras really are appended: the query blocks of the chunk's first
    # frame border the previous chunk's last frame and gain safeguards
    oprm = oracle_params(_prm(wl))
    ref = oracle_routes({0: p32[0]}, g, cov, oprm, M - 6, 6, nbr)
    n_extra = [len(v[1]) for v in ref.values()]
    assert sum(x > 0 for x in n_extra) >= 6 and max(n_extra) >= 4


def _synthetic_p(H, N, M, seed, peaked=1.0, flat=False):
    r = np.random.default_rng(seed)
    if flat:
        return np.full((H, N, M), 1.0 / M, dtype=np.float32)
    x = r.standard_normal((H, N, M)) * peaked
    p = np.exp(x - x.max(axis=2, keepdims=True))
    return (p / p.sum(axis=2, keepdims=True)).astype(np.float32)


def _geom(N, M, seed, frac=0.5):
    r = np.random.default_rng(seed + 99)
    g = r.random((N, M)).astype(np.float32)
    g[r.random((N, M)) < frac] = 0.0
    cov = (r.random(N) < 0.5).astype(np.uint8)
    cov[0], cov[-1] = 1, 0
    return g, cov


@pytest.mark.parametrize("peaked", [3.0, 6.0])
def test_route_mass_threshold_binds_before_cap(lib, peaked):
    H, N, M = 3, 6, 700
    p32 = _synthetic_p(H, N, M, 1, peaked=peaked)
    g, cov = _geom(N, M, 1)
    prm = rbs.route_params(theta_cov=0.6, theta_unc=0.7, k_cov=200, k_unc=300)
    _run_case(p32, g, cov, prm, 650, 20)
    # the cut must have come from the mass, not the cap, on some rows
    o = ort.route_row(p32[0, 1], g[1], bool(cov[1]), oracle_params(prm), 650, 20)
    assert len(o[0]) < (200 if cov[1] else 300)


def test_route_exact_ties_go_to_lower_ids(lib):
    H, N, M = 2, 4, 300
    p32 = _synthetic_p(H, N, M, 2, flat=True)
    g = np.zeros((N, M), np.float32)
    g[:, [5, 77, 150, 299]] = [0.2, 1.0, 0.5, 0.3]   # all saturate: equal multipliers
    cov = np.array([1, 0, 1, 0], np.uint8)
    prm = rbs.route_params(theta_cov=2.0, theta_unc=2.0, k_cov=30, k_unc=40)
    _run_case(p32, g, cov, prm, 280, 10)


def test_route_g_at_tau_and_g_ref(lib):
    H, N, M = 1, 4, 64
    p32 = _synthetic_p(H, N, M, 3, flat=True)
    g = np.zeros((N, M), np.float32)
    g[:, 10] = np.float32(0.1)    # == tau: no boost (strict >)
    g[:, 11] = np.float32(0.2)    # == g_ref: full boost
    g[:, 12] = np.float32(0.15)   # partial
    g[:, 13] = np.nextafter(np.float32(0.1), np.float32(1))  # just above tau
    cov = np.ones(N, np.uint8)
    prm = rbs.route_params(theta_cov=2.0, k_cov=4)
    _run_case(p32, g, cov, prm, 62, 2)


@pytest.mark.parametrize("M,K,prev", [(5, 80, 2), (40, 10, 12), (100, 60, 0), (100, 0, 4),
                                      (20, 20, 20), (1, 5, 1), (3, 1, 0)])
def test_route_edge_budgets(lib, M, K, prev):
    H, N = 2, 3
    p32 = _synthetic_p(H, N, M, M + K)
    g, cov = _geom(N, M, M)
    prm = rbs.route_params(k_cov=K, k_unc=K)
    _run_case(p32, g, cov, prm, M - prev, prev)


def test_route_reserved_mass_reaches_theta(lib):
    H, N, M = 1, 2, 50
    p32 = np.full((H, N, M), 1e-4, np.float32)
    p32[:, :, 40:44] = (1 - 46e-4) / 4
    g, cov = _geom(N, M, 5)
    _run_case(p32, g, cov, rbs.route_params(), 40, 4)


def test_route_safeguards_and_references(lib):
    H, N, M = 2, 3, 120
    p32 = _synthetic_p(H, N, M, 6)
    g, cov = _geom(N, M, 6)
    nbr = [[0, 5, 119], [], [7, 7, 8, 110]]
    ref = (3, 5, 64, 64)
    prm = rbs.route_params(k_cov=20, k_unc=30)
    _run_case(p32, g, cov, prm, 110, 10, nbr=nbr, ref=ref)


def test_route_large_history_uses_workspace(lib):
    H, N, M = 1, 2, 13000
    p32 = _synthetic_p(H, N, M, 7)
    g, cov = _geom(N, M, 7)
    prm = rbs.route_params(k_cov=100, k_unc=1000)
    _run_case(p32, g, cov, prm, M - 48, 48)


def test_route_large_cap(lib):
    H, N, M = 1, 3, 5000
    p32 = _synthetic_p(H, N, M, 8)
    g, cov = _geom(N, M, 8)
    prm = rbs.route_params(theta_cov=2.0, theta_unc=0.95, k_cov=4096, k_unc=2500)
    _run_case(p32, g, cov, prm, 0, 64)


def test_route_bad_safeguard_ids_are_flagged(lib):
    H, N, M = 1, 2, 30
    p = torch.from_numpy(_synthetic_p(H, N, M, 9)).cuda()
    g = torch.zeros(N, M, device="cuda")
    cv = torch.zeros(N, dtype=torch.uint8, device="cuda")
    ref = torch.tensor([3, 31, -2], dtype=torch.int32, device="cuda")
    R = 10
    rid = torch.empty(H, N, R, dtype=torch.int32, device="cuda")
    rl = torch.empty(H, N, dtype=torch.int32, device="cuda")
    rn = torch.empty(H, N, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    prm = rbs.route_params(k_cov=5, k_unc=5, theta_unc=2.0)
    rbs.velox_route_build(p, g, cv, prm, 28, 2, None, None, 0, ref, 3, H, N, M, rid, rl, rn, R,
                          ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) & rbs.DEV_BAD_SAFEGUARD
    for i in range(N):
        ids = rid[0, i, :int(rl[0, i])].tolist()
        assert all(0 <= x < M for x in ids) and len(set(ids)) == len(ids)


def test_route_at_the_largest_history_and_cap(lib):
    # M = VELOX_MAX_BLOCKS = 65536 (keys in the workspace), caps at
    # VELOX_MAX_ROUTE = 4096 (the bitonic sort over 4096 survivors); covered
    # rows take the threshold above 1 (the cap binds), uncovered rows 0.9 on
    # peaked importance
    H, N, M = 1, 3, 65536
    p32 = _synthetic_p(H, N, M, 9, peaked=4.0)
    g, cov = _geom(N, M, 9)
    prm = rbs.route_params(theta_cov=2.0, theta_unc=0.9, k_cov=4096, k_unc=4096)
    _run_case(p32, g, cov, prm, M - 48, 48)
