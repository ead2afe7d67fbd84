"""Audit counts (R_geo, R_50, top-80 recall, changed blocks) on the GPU vs the
oracle: integer counts, bit-exact."""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from oracle import audit as oa
from oracle import route as ort
from synth import config, make_inputs
from parity import oracle_params

pytestmark = pytest.mark.gpu


def _gpu_counts(p, g, prm, k_geo, k_fuse):
    H, N, M = p.shape
    counts = torch.full((H, N, 6), -1, dtype=torch.int32, device="cuda")
    rbs.velox_route_audit(p, g, H, N, M, prm, k_geo, k_fuse, counts)
    torch.cuda.synchronize()
    return counts.cpu().numpy()


def _oracle_counts(p, g, prm, k_geo, k_fuse):
    return oa.audit(p.cpu().numpy(), g.cpu().numpy(), oracle_params(prm), k_geo, k_fuse)


def test_audit_config2_from_gpu_importance(lib):
    # the audit scale: 40 heads, 12 query blocks, 143 history blocks; p from
    # the library's own importance step, g with 10 % positive blocks
    wl = config(2)
    inp = make_inputs(wl, "cuda")
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    p = torch.empty(H, N, M, device="cuda")
    ws = torch.empty(rbs.velox_workspace_size(H, N, M, 128), dtype=torch.uint8, device="cuda")
    rbs.velox_block_importance(inp.Q, inp.K, H, N, M, 128, 128, 1.0, p, ws)
    prm = rbs.route_params(2.0, 0.1, 0.2, 0.9, 0.9, 80, 150)
    got = _gpu_counts(p, inp.g, prm, 50, 80)
    ref = _oracle_counts(p, inp.g, prm, 50, 80)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("H,N,M,kg,kf,lam", [(2, 3, 17, 5, 8, 2.0), (1, 4, 300, 50, 80, 2.0),
                                             (3, 2, 40, 50, 80, 0.0), (1, 2, 9, 3, 20, 1.5)])
def test_audit_random_with_ties(lib, H, N, M, kg, kf, lam):
    r = np.random.default_rng(H * 1000 + M)
    # few distinct values so that ranks tie often (ties go to the lower id)
    p = (r.integers(0, 6, size=(H, N, M)) / 8.0).astype(np.float32)
    g = np.where(r.random((N, M)) < 0.3, r.integers(0, 5, size=(N, M)) / 4.0, 0.0)
    p, g = torch.from_numpy(p).cuda(), torch.from_numpy(g.astype(np.float32)).cuda()
    prm = rbs.route_params(lam, 0.25, 0.5, 0.9, 0.9, 80, 150)
    assert np.array_equal(_gpu_counts(p, g, prm, kg, kf), _oracle_counts(p, g, prm, kg, kf))


def test_audit_largest_m_sampled_rows(lib):
    H, N, M = 2, 3, 4096
    r = np.random.default_rng(9)
    x = r.standard_normal((H, N, M))
    p = np.exp(x - x.max(-1, keepdims=True))
    p = (p / p.sum(-1, keepdims=True)).astype(np.float32)
    g = np.where(r.random((N, M)) < 0.1, 0.2 + 0.8 * r.random((N, M)), 0.0).astype(np.float32)
    prm = rbs.route_params(2.0, 0.1, 0.2, 0.9, 0.9, 80, 150)
    got = _gpu_counts(torch.from_numpy(p).cuda(), torch.from_numpy(g).cuda(), prm, 50, 80)
    op = oracle_params(prm)
    for h, i in ((0, 0), (1, 2)):
        assert np.array_equal(got[h, i], oa.audit_row(p[h, i], g[i], op, 50, 80))


def test_audit_host_validation(lib):
    p = torch.zeros(1, 1, 4097, device="cuda")
    g = torch.zeros(1, 4097, device="cuda")
    c = torch.zeros(1, 1, 6, dtype=torch.int32, device="cuda")
    prm = rbs.route_params(2.0, 0.1, 0.2, 0.9, 0.9, 80, 150)
    with pytest.raises(rbs.VeloxError):
        rbs.velox_route_audit(p, g, 1, 1, 4097, prm, 50, 80, c)
    with pytest.raises(rbs.VeloxError):
        rbs.velox_route_audit(p, g, 1, 1, 16, prm, 0, 80, c)
