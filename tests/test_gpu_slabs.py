"""Slab-table build, multiwarp and the whole geometry chain on the GPU vs the
fp64 oracle.

Slab tables: rectangles, cameras and flags exact, and the percentiles
bit-exact (both sides interpolate the order statistics of the fp32 samples
in fp64 and round once to fp32: the reading of "10/90 percentile" fixes the
precision).  Multiwarp: the landing token of a sample is an integer decided
by floats; tokens that no marginal sample touches must have the oracle's
hole pattern and depths within MW_RTOL (tests/parity.py), and the marginal
ones are counted and bounded.  The chain test checks every stage against
the oracle applied to that stage's own GPU inputs, so the margins of one
stage do not leak into the next."""

import numpy as np
import pytest
import torch

import routed_block_sparse_b200 as rbs
from oracle import geometry as geo
from oracle import gilbert
from oracle import slabs as osl
from parity import check_coverage_bounds, check_g_bounds, check_multiwarp
from synth.depth import make_rollout
from synth.geometry import pack_slabs

pytestmark = pytest.mark.gpu


def _order(T, H, W, b, nc, layout):
    n = nc * T * H * W
    cell = torch.empty(n, dtype=torch.int32, device="cuda")
    fn = rbs.velox_gilbert_order if layout == "gilbert" else rbs.velox_thw_linear_order
    fn(T, H, W, nc, b, cell_of_rank=cell)
    return cell


def _gpu_slabs(depth, conf, mask, frame_base, H, W, s, cell, b, first, n, prm, uvz=False):
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = torch.full((n, 8), -5, dtype=torch.int32, device="cuda")
    tok = torch.full((n, b, 3), -1.0, device="cuda") if uvz else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_slab_table(dev(depth), dev(conf), dev(mask), depth.shape[0], frame_base, H, W, s,
                         cell, cell.numel(), b, first, n, prm.c_min, prm.n_min, prm.p_lo,
                         prm.p_hi, out, st, token_uvz=tok)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    return (o[:, :6].view(np.float32), o[:, 6], o[:, 7], int(st.item()),
            None if tok is None else tok.cpu().numpy())


@pytest.mark.parametrize("layout,s", [("gilbert", 1), ("gilbert", 2), ("thw", 1), ("thw", 3)])
def test_slab_table_matches_oracle(lib, layout, s):
    T, H, W, b, nc = 4, 8, 16, 32, 3
    r = make_rollout(5, nc * T, H, W, s)
    cell = _order(T, H, W, b, nc, layout)
    prm = osl.SlabParams(s=s, c_min=0.5, n_min=6 * s * s)
    n = nc * T * H * W // b
    slab, cam, valid, st, _ = _gpu_slabs(r.depth, r.conf, r.mask, 0, H, W, s, cell, b, 0, n, prm)
    ref = osl.slab_table(r.depth, r.conf, r.mask, cell.cpu().numpy(), H, W, b, 0, 0, n, prm)
    assert st == 0
    assert np.array_equal(slab, ref[0]) and np.array_equal(cam, ref[1])
    assert np.array_equal(valid, ref[2])
    assert valid.mean() > 0.5


def test_slab_table_chunk48_history_and_window(lib):
    # chunk-48 lattice: the 2256 history blocks of chunks 0..46 from 188 frames
    T, H, W, b, nc = 4, 32, 48, 128, 48
    r = make_rollout(7, 47 * T, H, W, 1)
    cell = _order(T, H, W, b, nc, "gilbert")
    prm = osl.SlabParams(s=1)
    slab, cam, valid, st, _ = _gpu_slabs(r.depth, r.conf, r.mask, 0, H, W, 1, cell, b, 0, 2256,
                                         prm)
    assert st == 0
    cr = cell.cpu().numpy()
    pick = [0, 1, 11, 12, 1000, 2255]
    for j in pick:
        ref = osl.slab_table(r.depth, r.conf, r.mask, cr, H, W, b, 0, j, 1, prm)
        assert np.array_equal(slab[j], ref[0][0]) and cam[j] == ref[1][0] and valid[j] == ref[2][0]
    # a window of frames 100..139 and blocks inside it
    sub = r.depth[100:140]
    s2, c2, v2, st2, _ = _gpu_slabs(sub, None, None, 100, H, W, 1, cell, b, 1200, 300, prm)
    ref = osl.slab_table(sub, None, None, cr, H, W, b, 100, 1200, 300, prm)
    assert st2 == 0 and np.array_equal(s2, ref[0]) and np.array_equal(v2, ref[2])


def test_slab_table_flags_blocks_outside_the_frames(lib):
    T, H, W, b, nc = 2, 4, 8, 8, 2
    r = make_rollout(2, 2, H, W, 1)          # frames 0..1 only
    cell = _order(T, H, W, b, nc, "gilbert")
    prm = osl.SlabParams(s=1, n_min=1)
    # blocks 0..15: frames 0..3, of which only 0..1 are given
    slab, _, valid, st, _ = _gpu_slabs(r.depth, None, None, 0, H, W, 1, cell, b, 0, 16, prm)
    assert st & rbs.DEV_BAD_CELL
    assert np.all(valid[8:] == 0) and np.all(slab[8:] == 0)
    ref = osl.slab_table(r.depth, None, None, cell.cpu().numpy(), H, W, b, 0, 0, 8, prm)
    assert np.array_equal(slab[:8], ref[0])


def _gpu_multiwarp(cams, src_depth, src_cam, tgt_cam, H, W, s, k_warp):
    zq = torch.full((len(tgt_cam), H, W), -1.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(rbs.velox_multiwarp_workspace_size(len(src_cam), len(tgt_cam), H, W),
                     dtype=torch.uint8, device="cuda")
    rbs.velox_multiwarp(torch.from_numpy(cams).cuda(), cams.shape[0],
                        torch.from_numpy(np.ascontiguousarray(src_depth)).cuda(),
                        torch.tensor(src_cam, dtype=torch.int32, device="cuda"), len(src_cam),
                        torch.tensor(tgt_cam, dtype=torch.int32, device="cuda"), len(tgt_cam),
                        H, W, s, k_warp, zq, ws, st)
    torch.cuda.synchronize()
    return zq.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("H,W,s,k", [(8, 16, 2, 2), (6, 10, 3, 2), (8, 16, 1, 1), (8, 16, 2, 5)])
def test_multiwarp_matches_oracle(lib, H, W, s, k):
    r = make_rollout(3, 40, H, W, s, step=0.05)
    src = [37, 36, 30, 29, 20, 19]            # newest first
    tgt = [39, 38]
    zq, st = _gpu_multiwarp(r.cams, r.depth[src], src, tgt, H, W, s, k)
    assert st == 0
    for j, t in enumerate(tgt):
        ref, unsure = osl.multiwarp_bounds(r.cams, r.depth[src], src, t, H, W, s, k)
        check_multiwarp(zq[j], ref, unsure)
    if k <= s * s:  # s x s samples per source token: k_warp above that rarely holds
        assert (zq > 0).mean() > 0.3


def test_multiwarp_chunk48_frame(lib):
    H, W, s = 32, 48, 2
    r = make_rollout(4, 192, H, W, s)
    src = [183, 180, 179, 176]
    zq, st = _gpu_multiwarp(r.cams, r.depth[src], src, [188], H, W, s, 2)
    ref, unsure = osl.multiwarp_bounds(r.cams, r.depth[src], src, 188, H, W, s, 2)
    assert st == 0 and (ref > 0).mean() > 0.9
    check_multiwarp(zq[0], ref, unsure)


def test_multiwarp_bad_camera_is_flagged(lib):
    H, W, s = 4, 8, 2
    r = make_rollout(1, 4, H, W, s)
    zq, st = _gpu_multiwarp(r.cams, r.depth[[1, 2]], [99, 2], [3], H, W, s, 2)
    assert st & rbs.DEV_BAD_CAMERA
    ref, unsure = osl.multiwarp_bounds(r.cams, r.depth[[2]], [2], 3, H, W, s, 2)
    check_multiwarp(zq[0], ref, unsure)


def test_geometry_chain_depth_to_g_and_coverage(lib):
    """Depth maps -> history slab table -> multiwarp query depth -> query slabs
    and tokens -> slab overlap and coverage: every GPU stage against the
    oracle applied to that stage's GPU inputs."""
    T, H, W, b, nc, s = 4, 8, 16, 32, 6, 2
    q_chunk = nc - 1
    r = make_rollout(11, nc * T, H, W, s, step=0.05)
    cell = _order(T, H, W, b, nc, "gilbert")
    cr = cell.cpu().numpy()
    per_chunk = T * H * W // b
    M = q_chunk * per_chunk
    hist_frames = q_chunk * T
    prm = osl.SlabParams(s=s, n_min=16)
    hs, hc, hv, st, _ = _gpu_slabs(r.depth[:hist_frames], r.conf[:hist_frames],
                                   r.mask[:hist_frames], 0, H, W, s, cell, b, 0, M, prm)
    assert st == 0
    ref_h = osl.slab_table(r.depth[:hist_frames], r.conf[:hist_frames], r.mask[:hist_frames], cr,
                           H, W, b, 0, 0, M, prm)
    assert np.array_equal(hs, ref_h[0]) and np.array_equal(hc, ref_h[1])
    assert np.array_equal(hv, ref_h[2])
    # query depth of the current chunk's frames from the newest history frames
    src = list(range(hist_frames - 1, hist_frames - 9, -1))
    tgt = list(range(hist_frames, hist_frames + T))
    zq, st = _gpu_multiwarp(r.cams, r.depth[src], src, tgt, H, W, s, 2)
    assert st == 0
    for j, t in enumerate(tgt):
        ref, unsure = osl.multiwarp_bounds(r.cams, r.depth[src], src, t, H, W, s, 2)
        check_multiwarp(zq[j], ref, unsure)
    # query slabs and tokens from the GPU's multiwarp depth
    qprm = osl.SlabParams(s=1, n_min=8)
    first_q = q_chunk * per_chunk
    qs, qc, qv, st, quvz = _gpu_slabs(zq, None, None, hist_frames, H, W, 1, cell, b, first_q,
                                      per_chunk, qprm, uvz=True)
    assert st == 0
    ref_q = osl.slab_table(zq, None, None, cr, H, W, b, hist_frames, first_q, per_chunk, qprm)
    assert np.array_equal(qs, ref_q[0]) and np.array_equal(qc, ref_q[1])
    assert np.array_equal(qv, ref_q[2])
    ref_uvz = osl.block_tokens(zq, None, None, cr, H, W, b, hist_frames, first_q, per_chunk)
    assert np.array_equal(quvz, ref_uvz)
    # overlap and coverage on the chain's slabs (query slabs kept valid: the
    # overlap of a query block is defined whatever its own n_min)
    cams = torch.from_numpy(r.cams).cuda()
    qpack = torch.from_numpy(pack_slabs(qs, qc)).cuda()
    hpack = torch.from_numpy(pack_slabs(hs, hc, hv)).cuda()
    N = per_chunk
    g = torch.empty(N, M, device="cuda")
    stt = torch.zeros(1, dtype=torch.int32, device="cuda")
    rbs.velox_slab_overlap(cams, cams.shape[0], qpack, N, hpack, M, 8, g, stt)
    rho = torch.empty(N, device="cuda")
    cov = torch.empty(N, dtype=torch.uint8, device="cuda")
    rbs.velox_coverage(cams, cams.shape[0], qpack, torch.from_numpy(quvz).cuda(), N, b, hpack, M,
                       0.9, rho, cov, stt)
    torch.cuda.synchronize()
    assert int(stt.item()) == 0
    g_ref, g_lo, g_hi = geo.overlap_bounds(r.cams, qc, qs, hc, hs, hv, 8)
    assert (g_ref > 0).any()
    check_g_bounds(g.cpu().numpy().astype(np.float64), g_ref, g_lo, g_hi)
    n, n_lo, n_hi = geo.coverage_bounds(r.cams, qc, quvz, hc, hs, hv)
    check_coverage_bounds(rho.cpu().numpy(), cov.cpu().numpy(), n, n_lo, n_hi, b, 0.9)


@pytest.mark.parametrize("seed", range(6))
def test_multiwarp_random_poses(lib, seed):
    # sources and target from cameras rotated up to 0.6 rad about random
    # axes with different intrinsics; depths uniform in [2, 8] with holes
    from synth.geometry import random_depth_maps, random_pose_scene
    H, W = 8, 16
    s = 1 + seed % 2
    k = 1 + seed % 3
    cams = random_pose_scene(seed, 1, 1, frame_hw=(H, W), n_cams=5).cams
    src = [4, 3, 2, 1]                        # newest first
    depth = random_depth_maps(seed, len(src), H, W, s)
    zq, st = _gpu_multiwarp(cams, depth, src, [0], H, W, s, k)
    assert st == 0
    ref, unsure = osl.multiwarp_bounds(cams, depth, src, 0, H, W, s, k)
    check_multiwarp(zq[0], ref, unsure)
