"""Slab overlap g and coverage rho on the GPU vs the fp64 oracle.

Inside counts and covered-token counts must agree exactly wherever the
oracle's decisions are clear of its marginal distance, and lie within the
oracle's [lo, hi] range where some decision is marginal (tests/parity.py)."""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from oracle import geometry as geo
from parity import check_coverage_bounds, check_g_bounds
from synth.geometry import make_scene, pack_slabs

pytestmark = pytest.mark.gpu


def _dev(scene, q_cam=None, h_cam=None):
    q_cam = scene.q_cam if q_cam is None else q_cam
    h_cam = scene.h_cam if h_cam is None else h_cam
    cams = torch.from_numpy(scene.cams).cuda()
    qs = torch.from_numpy(pack_slabs(scene.q_slab, q_cam)).cuda()
    hs = torch.from_numpy(pack_slabs(scene.h_slab, h_cam, scene.h_valid)).cuda()
    return cams, qs, hs


def _overlap(scene, G, q_cam=None, h_cam=None):
    cams, qs, hs = _dev(scene, q_cam, h_cam)
    N, M = qs.shape[0], hs.shape[0]
    g = torch.full((N, M), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_slab_overlap(cams, cams.shape[0], qs, N, hs, M, G, g, st)
    torch.cuda.synchronize()
    return g.cpu().numpy().astype(np.float64), int(st.item())


def _coverage(scene, eta=0.9, q_cam=None, h_cam=None):
    cams, qs, hs = _dev(scene, q_cam, h_cam)
    N, M, b = qs.shape[0], hs.shape[0], scene.q_uvz.shape[1]
    uvz = torch.from_numpy(np.ascontiguousarray(scene.q_uvz)).cuda()
    rho = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    cov = torch.full((N,), 7, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_coverage(cams, cams.shape[0], qs, uvz, N, b, hs, M, eta, rho, cov, st)
    torch.cuda.synchronize()
    return rho.cpu().numpy(), cov.cpu().numpy(), int(st.item())


def _bounds(s, G, q_cam=None, h_cam=None):
    q_cam = s.q_cam if q_cam is None else q_cam
    h_cam = s.h_cam if h_cam is None else h_cam
    return geo.overlap_bounds(s.cams, q_cam, s.q_slab, h_cam, s.h_slab, s.h_valid, G)


@pytest.mark.parametrize("seed,N,M,G", [(1, 6, 40, 4), (2, 13, 29, 8), (3, 4, 24, 1),
                                        (4, 3, 17, 5)])
def test_overlap_small(lib, seed, N, M, G):
    s = make_scene(seed, N, M)
    g, st = _overlap(s, G)
    assert st == 0
    ref, lo, hi = _bounds(s, G)
    assert (ref > 0).any() and (ref == 0).any()
    check_g_bounds(g, ref, lo, hi)


def test_overlap_identical_slab_is_one(lib):
    # every query slab against itself (same camera, valid): IoU 1 exactly
    s = make_scene(9, 5, 5)
    s.h_slab, s.h_cam, s.h_valid = s.q_slab.copy(), s.q_cam.copy(), np.ones(5, np.int32)
    g, st = _overlap(s, 8)
    assert st == 0 and np.all(np.diag(g) == 1.0)


@pytest.mark.slow
def test_overlap_chunk48_sampled(lib):
    # chunk-48 shape: 48 query blocks against 2256 history blocks, 8^3 samples
    s = make_scene(20261203, 48, 2256)
    g, st = _overlap(s, 8)
    assert st == 0 and np.all((g >= 0) & (g <= 1))
    assert np.all(g[:, s.h_valid == 0] == 0)
    rng = np.random.default_rng(5)
    nz = np.argwhere(g > 0)
    z = np.argwhere(g == 0)
    pick = np.concatenate([nz[rng.choice(len(nz), 48, replace=False)],
                           z[rng.choice(len(z), 16, replace=False)]])
    ref, lo, hi = (np.zeros(len(pick)) for _ in range(3))
    for k, (i, r) in enumerate(pick):
        n, n_lo, n_hi, vi, vr = geo.slab_iou_counts(s.cams[s.q_cam[i]], s.q_slab[i],
                                                    s.cams[s.h_cam[r]], s.h_slab[r],
                                                    bool(s.h_valid[r]), 8)
        ref[k], lo[k], hi[k] = (geo.iou_from_count(c, vi, vr, 8) for c in (n, n_lo, n_hi))
    check_g_bounds(np.array([g[i, r] for i, r in pick]), ref, lo, hi)


@pytest.mark.parametrize("seed,N,M,b", [(1, 12, 40, 128), (2, 7, 31, 50), (3, 5, 12, 1)])
def test_coverage_small(lib, seed, N, M, b):
    s = make_scene(seed, N, M, b)
    rho, cov, st = _coverage(s)
    assert st == 0
    n, lo, hi = geo.coverage_bounds(s.cams, s.q_cam, s.q_uvz, s.h_cam, s.h_slab, s.h_valid)
    check_coverage_bounds(rho, cov, n, lo, hi, b, 0.9)


def test_coverage_threshold_edges(lib):
    s = make_scene(1, 12, 40)
    rho, _, _ = _coverage(s)
    for eta in (0.0, float(rho[3]), 1.0, 1.5):
        _, cov, st = _coverage(s, eta)
        assert st == 0
        assert np.array_equal(cov, (rho >= np.float32(eta)).astype(np.uint8))


@pytest.mark.slow
def test_coverage_chunk48_sampled(lib):
    s = make_scene(20261203, 48, 2256)
    rho, cov, st = _coverage(s)
    assert st == 0
    assert np.all(cov == (rho >= np.float32(0.9)))
    pick = [0, 17, 47]
    n, lo, hi = geo.coverage_bounds(s.cams, s.q_cam[pick], s.q_uvz[pick], s.h_cam, s.h_slab,
                                    s.h_valid)
    check_coverage_bounds(rho[pick], cov[pick], n, lo, hi, 128, 0.9)


def test_bad_camera_is_flagged_not_read(lib):
    s = make_scene(4, 6, 30)
    h_cam = s.h_cam.copy()
    h_cam[3] = s.n_cams          # out of range
    s.h_valid[3] = 1
    g, st = _overlap(s, 4, h_cam=h_cam)
    assert st & rbs.DEV_BAD_CAMERA
    assert np.all(g[:, 3] == 0)
    ref, lo, hi = _bounds(s, 4)
    keep = np.ones(30, bool)
    keep[3] = False
    check_g_bounds(g[:, keep], ref[:, keep], lo[:, keep], hi[:, keep])
    q_cam = s.q_cam.copy()
    q_cam[2] = -1
    rho, cov, st = _coverage(s, q_cam=q_cam)
    assert st & rbs.DEV_BAD_CAMERA and rho[2] == 0 and cov[2] == 0


def test_host_validation(lib):
    s = make_scene(1, 2, 4)
    cams, qs, hs = _dev(s)
    g = torch.zeros(2, 4, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(rbs.VeloxError):
        rbs.velox_slab_overlap(cams, cams.shape[0], qs, 2, hs, 4, 33, g, st)
    with pytest.raises(rbs.VeloxError):
        rbs.velox_slab_overlap(cams, cams.shape[0], qs, 0, hs, 4, 8, g, st)
    uvz = torch.zeros(2, 129, 3, device="cuda")
    rho = torch.zeros(2, device="cuda")
    cov = torch.zeros(2, dtype=torch.uint8, device="cuda")
    with pytest.raises(rbs.VeloxError):
        rbs.velox_coverage(cams, cams.shape[0], qs, uvz, 2, 129, hs, 4, 0.9, rho, cov, st)


@pytest.mark.parametrize("seed", range(8))
def test_random_poses_overlap_and_coverage(lib, seed):
    # arbitrary rotations (up to 0.6 rad about random axes), focal lengths,
    # principal points, rectangles and depth ranges: g and the covered counts
    # against the fp64 oracle under the marginal-decision rule
    from synth.geometry import random_pose_scene
    s = random_pose_scene(seed, 7, 60, b=64)
    G = (2, 4, 8)[seed % 3]
    g, st = _overlap(s, G)
    assert st == 0
    ref, lo, hi = _bounds(s, G)
    check_g_bounds(g, ref, lo, hi)
    rho, cov, st = _coverage(s, eta=0.5)
    assert st == 0
    n, nlo, nhi = geo.coverage_bounds(s.cams, s.q_cam, s.q_uvz, s.h_cam, s.h_slab, s.h_valid)
    check_coverage_bounds(rho, cov, n, nlo, nhi, 64, 0.5)

