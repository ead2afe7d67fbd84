"""Pins of the slab-table and multiwarp oracle.

Percentiles against numpy's linear-interpolation percentile and the integer
closed form; block rectangles against the bounding boxes of the order's own
block map; reliability filtering and n_min; multiwarp closed forms: an
identity warp returns the source depth (k_warp = 1) or the median of a
token's s x s samples, a forward move towards a fronto-parallel plane lowers
every depth by the move, a sideways move by a whole number of tokens shifts
the map, the newest source that gives k_warp samples wins, and too few
samples leave holes.
"""

import numpy as np
import pytest

from oracle import gilbert
from oracle import slabs as osl


def cam(fx=4.0, fy=4.0, cx=4.0, cy=2.0, C=(0.0, 0.0, 0.0)):
    return np.array([fx, fy, cx, cy, *np.eye(3).reshape(-1), *C], dtype=np.float32)


def test_percentile_matches_numpy_and_closed_form():
    assert osl.percentile_sorted(list(range(11)), 0.1) == 1.0
    assert osl.percentile_sorted(list(range(11)), 0.9) == 9.0
    assert osl.percentile_sorted([3.0], 0.9) == 3.0
    rng = np.random.default_rng(0)
    for n in (2, 3, 7, 128, 511):
        v = np.sort(rng.standard_normal(n))
        for q in (0.1, 0.5, 0.9):
            ref = np.percentile(v, 100 * q)
            assert abs(osl.percentile_sorted(v.tolist(), q) - ref) <= 1e-14 * (1 + abs(ref))


@pytest.mark.parametrize("layout", ["gilbert", "thw"])
def test_rectangles_are_block_bounding_boxes(layout):
    T, H, W, b, nc = 2, 4, 8, 8, 2
    order = gilbert.global_order if layout == "gilbert" else gilbert.thw_linear_order
    _, cell, block = order(T, H, W, nc, b)
    n_frames = nc * T
    depth = np.full((n_frames, H, W), 3.0, dtype=np.float32)
    n_blocks = n_frames * H * W // b
    slab, camv, valid = osl.slab_table(depth, None, None, cell, H, W, b, 0, 0, n_blocks,
                                       osl.SlabParams(s=1, n_min=1))
    blk = block.reshape(n_frames, H, W)
    for r in range(n_blocks):
        f, ys, xs = np.nonzero(blk == r)
        assert valid[r] == 1 and camv[r] == f[0]
        assert slab[r].tolist() == [xs.min(), xs.max() + 1, ys.min(), ys.max() + 1, 3.0, 3.0]


def test_reliability_and_percentiles_with_subsamples():
    T, H, W, b, nc, s = 1, 2, 4, 4, 1, 2
    _, cell, _ = gilbert.thw_linear_order(T, H, W, nc, b)   # block 0: row 0, block 1: row 1
    depth = np.zeros((1, H * s, W * s), dtype=np.float32)
    conf = np.ones_like(depth)
    mask = np.ones(depth.shape, dtype=np.uint8)
    # block 0: 16 samples 1..16, the 4 largest unreliable (low confidence)
    depth[0, :2, :] = np.arange(1, 17, dtype=np.float32).reshape(2, 8)
    conf[0, 1, 4:] = 0.1
    # block 1: only 3 reliable samples (the rest masked out or at depth 0)
    depth[0, 2:, :] = 5.0
    mask[0, 2:, :] = 0
    mask[0, 2, :3] = 1
    slab, _, valid = osl.slab_table(depth, conf, mask, cell, H, W, b, 0, 0, 2,
                                    osl.SlabParams(s=s, c_min=0.5, n_min=4))
    rel = np.sort(np.concatenate([np.arange(1, 9), np.arange(9, 13)]).astype(np.float64))
    assert valid.tolist() == [1, 0]
    assert slab[0, 4] == np.float32(np.percentile(rel, 10))
    assert slab[0, 5] == np.float32(np.percentile(rel, 90))
    assert slab[1].tolist() == [0.0] * 6


def test_identity_warp_returns_depth_or_sample_median():
    H, W = 4, 8
    c = cam()
    rng = np.random.default_rng(1)
    d = rng.uniform(1.0, 3.0, size=(1, H, W)).astype(np.float32)
    zq = osl.multiwarp([c], d, [0], 0, H, W, s=1, k_warp=1)
    assert np.array_equal(zq, d[0])
    assert np.all(osl.multiwarp([c], d, [0], 0, H, W, s=1, k_warp=2) == 0)
    d2 = rng.uniform(1.0, 3.0, size=(1, 2 * H, 2 * W)).astype(np.float32)
    zq = osl.multiwarp([c], d2, [0], 0, H, W, s=2, k_warp=2)
    blocks = d2[0].reshape(H, 2, W, 2).transpose(0, 2, 1, 3).reshape(H, W, 4).astype(np.float64)
    assert np.array_equal(zq, np.median(blocks, axis=-1).astype(np.float32))


def test_forward_move_towards_a_plane():
    H, W, Z, dz = 4, 8, 4.0, 1.0
    src, tgt = cam(), cam(C=(0.0, 0.0, dz))
    d = np.full((1, 2 * H, 2 * W), Z, dtype=np.float32)
    zq = osl.multiwarp([src, tgt], d, [0], 1, H, W, s=2, k_warp=2)
    hit = zq > 0
    assert hit.sum() >= H * W // 2
    assert np.all(zq[hit] == Z - dz)


def test_sideways_whole_token_shift_and_recency():
    H, W, Z = 4, 8, 4.0
    # move right by 2 world units: at depth 4 with fx = 4 that is 2 tokens
    src, tgt = cam(), cam(C=(2.0, 0.0, 0.0))
    d_new = np.full((2, H, W), Z, dtype=np.float32)
    d_new[1] = 2.0 * Z                     # an older source at another depth
    zq = osl.multiwarp([src, tgt], d_new, [0, 0], 1, H, W, s=1, k_warp=1)
    # newest source: token x lands on x - 2; older source (twice as deep):
    # token x lands on x - 1, so it fills column W - 2 only; W - 1 stays a hole
    assert np.all(zq[:, :W - 2] == Z) and np.all(zq[:, W - 2] == 2.0 * Z)
    assert np.all(zq[:, W - 1] == 0)
    # the newest source gives every token one sample only: with k_warp = 2
    # nothing qualifies and the tokens stay holes
    assert np.all(osl.multiwarp([src, tgt], d_new, [0, 0], 1, H, W, s=1, k_warp=2) == 0)


def test_block_tokens_on_a_hand_built_lattice():
    # one frame (global frame 1) of H = 2, W = 4 tokens, s = 1; blocks of 4
    # tokens in an arbitrary rank order.  Cell index = (f H + y) W + x.
    H, W, b = 2, 4, 4
    f = 1
    order = [(1, 0), (0, 0), (0, 1), (1, 1),       # block 2: ranks 8..11 as (x, y)
             (3, 1), (2, 1), (2, 0), (3, 0)]       # block 3: ranks 12..15
    cell_of_rank = np.full(16, -1, dtype=np.int64)
    for k, (x, y) in enumerate(order):
        cell_of_rank[8 + k] = (f * H + y) * W + x
    depth = np.array([[[1.0, 2.0, 0.0, 4.0],
                       [5.0, -1.0, 7.0, 8.0]]], dtype=np.float32)
    mask = np.array([[[1, 1, 1, 1], [1, 1, 1, 0]]], dtype=np.uint8)    # (3, 1) masked
    conf = np.array([[[0.9, 0.4, 0.9, 0.9], [0.9, 0.9, 0.5, 0.9]]], dtype=np.float32)
    out = osl.block_tokens(depth, conf, mask, cell_of_rank, H, W, b, frame_base=1,
                           first_block=2, n_blocks=2, c_min=0.5)
    # (x + 0.5, y + 0.5, depth), depth 0 when the sample is not reliable:
    # (1, 0) conf 0.4 < 0.5; (1, 1) depth -1; (2, 0) depth 0; (3, 1) masked;
    # (2, 1) conf exactly 0.5 is kept
    want = [[[1.5, 0.5, 0.0], [0.5, 0.5, 1.0], [0.5, 1.5, 5.0], [1.5, 1.5, 0.0]],
            [[3.5, 1.5, 0.0], [2.5, 1.5, 7.0], [2.5, 0.5, 0.0], [3.5, 0.5, 4.0]]]
    assert out.dtype == np.float32 and out.tolist() == want
    # no confidence or mask given: only the depth decides
    out = osl.block_tokens(depth, None, None, cell_of_rank, H, W, b, 1, 2, 2)
    assert out[0, 0, 2] == 2.0 and out[1, 0, 2] == 8.0 and out[0, 3, 2] == 0.0


def test_samples_landing_on_token_edges_are_unsure():
    H, W, Z = 4, 8, 4.0
    d = np.full((1, H, W), Z, dtype=np.float32)
    # a sideways move of 0.5 world units at depth 4, fx = 4: half a token.
    # Token centres x + 0.5 land on x exactly: every landing is on an edge.
    src, tgt = cam(), cam(C=(0.5, 0.0, 0.0))
    zq, unsure = osl.multiwarp_bounds([src, tgt], d, [0], 1, H, W, s=1, k_warp=1)
    assert unsure.all()
    # a quarter of a token: token x lands at x + 0.25, a quarter token from
    # the nearest edge, in its own cell
    zq, unsure = osl.multiwarp_bounds([src, cam(C=(0.25, 0.0, 0.0))], d, [0], 1, H, W, s=1,
                                      k_warp=1)
    assert not unsure.any()
    assert np.all(zq == Z)


def test_warp_sample_closed_form():
    # forward move by 1 towards depth 4: depth 3, same pixel for the principal
    # ray, and the landing cell with its distance to the nearest token edge
    cell, depth, margin, cand = osl.warp_sample(cam(), cam(C=(0.0, 0.0, 1.0)), 4.5, 2.5, 4.0,
                                                4, 8)
    # u' = (4.5 - 4) * 4 / 3 + 4 = 4.666..., v' = (2.5 - 2) * 4 / 3 + 2 = 2.666...
    assert cell == (4, 2) and depth == 3.0 and cand == [(4, 2)]
    assert abs(margin - (1.0 / 3.0) * 3.0 / 4.0) < 1e-12
    # behind the target camera: no landing
    cell, depth, _, _ = osl.warp_sample(cam(), cam(C=(0.0, 0.0, 5.0)), 4.5, 2.5, 4.0, 4, 8)
    assert cell is None and depth < 0


def test_slab_needs_exactly_n_min_reliable_samples():
    # block 0 has exactly n_min reliable samples (valid), block 1 one fewer
    T, H, W, b, nc = 1, 2, 4, 4, 1
    _, cell, _ = gilbert.thw_linear_order(T, H, W, nc, b)
    depth = np.full((1, H, W), 2.0, dtype=np.float32)
    mask = np.ones(depth.shape, dtype=np.uint8)
    mask[0, 1, 0] = 0                     # row 1 (block 1): 3 reliable samples
    slab, _, valid = osl.slab_table(depth, None, mask, cell, H, W, b, 0, 0, 2,
                                    osl.SlabParams(s=1, n_min=4))
    assert valid.tolist() == [1, 0]
    assert slab[0].tolist() == [0.0, 4.0, 0.0, 1.0, 2.0, 2.0]


def test_a_marginal_landing_makes_both_neighbours_unsure():
    # one valid sample, moved half a token sideways: it lands exactly on the
    # edge between target tokens 2 and 3 of row 1, so either may receive it
    # in another precision; nothing else is unsure
    H, W, Z = 4, 8, 4.0
    d = np.zeros((1, H, W), dtype=np.float32)
    d[0, 1, 3] = Z
    src, tgt = cam(), cam(C=(0.5, 0.0, 0.0))
    zq, unsure = osl.multiwarp_bounds([src, tgt], d, [0], 1, H, W, s=1, k_warp=1)
    assert sorted(zip(*np.nonzero(unsure))) == [(1, 2), (1, 3)]
