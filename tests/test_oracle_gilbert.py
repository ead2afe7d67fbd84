"""Pins of the oracle's Gilbert order and neighbour safeguards.

What these check comes from the pages and from mathematics, not from the
oracle itself:

* the curve is a generalised Hilbert curve: on 2^k x 2^k frames it must be the
  textbook Hilbert curve (the classic d -> (x, y) map, written here from its
  usual rotate-and-reflect description);
* every cell is visited once, with unit lattice steps, across frame, block
  and chunk seams (Velox project page, "02 · Method", "Keeping neighbours
  adjacent in the block order");
* each chunk's ranks are contiguous (the order is "global-aligned");
* for chunks of an odd number of frames, chunk 1 is the horizontal mirror of
  chunk 0, and a plain per-chunk repeat breaks the seam (project page, figure
  "Incremental Gilbert order", toy case H=3, W=4, block 2, 3 frames);
* the safeguard table equals an O(n^2) brute force over token pairs.
"""

import itertools

import numpy as np
import pytest

from oracle import gilbert


def hilbert_d2xy(n, d):
    """Textbook Hilbert curve: position of step d on an n x n grid (n = 2^k)."""
    x = y = 0
    s = 1
    t = d
    while s < n:
        rx = 1 & (t // 2)
        ry = 1 & (t ^ rx)
        if ry == 0:
            if rx == 1:
                x, y = s - 1 - x, s - 1 - y
            x, y = y, x
        x += s * rx
        y += s * ry
        t //= 4
        s *= 2
    return x, y


@pytest.mark.parametrize("k", range(0, 7))
def test_power_of_two_frame_is_textbook_hilbert(k):
    n = 2 ** k
    assert gilbert.frame_curve(n, n) == [hilbert_d2xy(n, d) for d in range(n * n)]


def _supported(W, H):
    return W >= H and not (W % 2 == 1 and H % 2 == 0)


def test_frame_curve_unit_steps_and_corners():
    for W in range(1, 41):
        for H in range(1, W + 1):
            if not _supported(W, H):
                continue
            c = gilbert.frame_curve(W, H)
            assert len(c) == W * H and len(set(c)) == W * H
            assert all(0 <= x < W and 0 <= y < H for x, y in c)
            assert c[0] == (0, 0) and c[-1] == (W - 1, 0), (W, H)
            for a, b in zip(c, c[1:]):
                assert abs(a[0] - b[0]) + abs(a[1] - b[1]) == 1, (W, H, a, b)


def test_odd_by_even_has_no_unit_path():
    # The checkerboard colours of (0,0) and (W-1,0) agree when W is odd, and a
    # Hamiltonian path over an even number of cells joins opposite colours:
    # the construction must then contain a non-unit step or a different end.
    for W in (3, 5, 7, 9):
        for H in (2, 4):
            if H > W:
                continue
            c = gilbert.frame_curve(W, H)
            unit = all(abs(a[0] - b[0]) + abs(a[1] - b[1]) == 1 for a, b in zip(c, c[1:]))
            assert not (unit and c[-1] == (W - 1, 0))
    with pytest.raises(ValueError):
        gilbert.check_supported(2, 2, 3, 2)
    with pytest.raises(ValueError):
        gilbert.check_supported(2, 4, 3, 2)     # W < H
    with pytest.raises(ValueError):
        gilbert.check_supported(3, 3, 4, 5)     # 36 % 5 != 0


def _coords(c, H, W):
    f, r = divmod(c, H * W)
    y, x = divmod(r, W)
    return f, y, x


LATTICES = [
    (3, 3, 4, 2, 2),      # the pages' toy case
    (3, 3, 4, 2, 3),
    (4, 3, 4, 2, 3),
    (1, 5, 5, 5, 4),
    (2, 4, 6, 8, 3),
    (4, 8, 12, 128, 3),
    (3, 1, 6, 2, 2),
]


@pytest.mark.parametrize("T,H,W,b,nc", LATTICES)
def test_global_order_is_a_unit_step_path(T, H, W, b, nc):
    rank, cell, block = gilbert.global_order(T, H, W, nc, b)
    n = nc * T * H * W
    assert sorted(rank.tolist()) == list(range(n))
    assert np.array_equal(rank[cell], np.arange(n))
    for k in range(n - 1):
        a = _coords(int(cell[k]), H, W)
        b_ = _coords(int(cell[k + 1]), H, W)
        assert sum(abs(u - v) for u, v in zip(a, b_)) == 1, (k, a, b_)
    assert np.array_equal(block, rank // b)


@pytest.mark.parametrize("T,H,W,b,nc", LATTICES)
def test_chunks_own_contiguous_ranks_and_blocks(T, H, W, b, nc):
    rank, _, block = gilbert.global_order(T, H, W, nc, b)
    per = T * H * W
    for c in range(nc):
        seg = rank[c * per:(c + 1) * per]
        assert seg.min() == c * per and seg.max() == (c + 1) * per - 1
        blk = np.unique(block[c * per:(c + 1) * per])
        assert blk.tolist() == list(range(c * per // b, (c + 1) * per // b))


def test_toy_odd_chunk_is_mirrored_and_plain_repeat_breaks():
    T, H, W, b = 3, 3, 4, 2
    rank, cell, _ = gilbert.global_order(T, H, W, 2, b)
    per = T * H * W
    r = rank.reshape(2, T, H, W) - np.arange(2)[:, None, None, None] * per
    assert np.array_equal(r[1], r[0][:, :, ::-1])
    # A plain repeat of chunk 0's map puts chunk 1's first cell on the far
    # side of the seam: not a unit step from chunk 0's last cell.
    last0 = _coords(int(cell[per - 1]), H, W)
    first_plain = _coords(int(cell[0]) + per, H, W)
    assert sum(abs(u - v) for u, v in zip(last0, first_plain)) > 1
    first_global = _coords(int(cell[per]), H, W)
    assert sum(abs(u - v) for u, v in zip(last0, first_global)) == 1


def _brute_neighbours(T, H, W, nc, b, q_chunk, first, M, block=None):
    if block is None:
        _, _, block = gilbert.global_order(T, H, W, nc, b)
    n = nc * T * H * W
    coords = [_coords(c, H, W) for c in range(n)]
    per = T * H * W // b
    out = []
    for i in range(per):
        qb = q_chunk * per + i
        found = set()
        for c1, c2 in itertools.product(range(n), range(n)):
            if block[c1] != qb:
                continue
            u = int(block[c2])
            if u == qb or not (first <= u < first + M):
                continue
            if max(abs(p - q) for p, q in zip(coords[c1], coords[c2])) <= 1:
                found.add(u - first)
        out.append(sorted(found))
    return out


@pytest.mark.parametrize("T,H,W,b,nc,qc,first,M", [
    (3, 3, 4, 2, 2, 1, 0, 18),        # toy: history = chunk 0
    (3, 3, 4, 2, 3, 2, 0, 36),
    (3, 3, 4, 2, 3, 2, 5, 31),        # cache holds only the most recent blocks
    (2, 2, 4, 4, 3, 1, 0, 12),        # cache also holds later blocks
    (2, 3, 3, 3, 3, 2, 2, 10),
])
def test_neighbours_match_token_pair_brute_force(T, H, W, b, nc, qc, first, M):
    got = gilbert.neighbour_blocks(T, H, W, nc, b, qc, first, M)
    assert got == _brute_neighbours(T, H, W, nc, b, qc, first, M)


def test_history_neighbours_lie_in_previous_chunk_last_frame():
    # With a history-only cache, the only lattice neighbours of the current
    # chunk sit in the previous chunk's last frame.
    T, H, W, b, nc = 4, 4, 8, 16, 4
    per = T * H * W // b
    qc = nc - 1
    M = qc * per
    nb = gilbert.neighbour_blocks(T, H, W, nc, b, qc, 0, M)
    rank, _, block = gilbert.global_order(T, H, W, nc, b)
    last_frame = qc * T - 1
    lf_blocks = set(block.reshape(nc * T, H, W)[last_frame].ravel().tolist())
    for lst in nb:
        assert set(lst) <= lf_blocks
    assert any(len(lst) for lst in nb)


def test_thw_linear_rank_is_the_cell_index():
    # (f * H + y) * W + x is exactly the cell index: the THW-linear rank map
    # is the identity, and a block is 128 (here b) consecutive raster cells
    for T, H, W, b, nc in ((3, 3, 4, 2, 2), (2, 5, 3, 5, 3)):
        rank, cell, block = gilbert.thw_linear_order(T, H, W, nc, b)
        n = nc * T * H * W
        assert np.array_equal(rank, np.arange(n)) and np.array_equal(cell, np.arange(n))
        assert np.array_equal(block, np.arange(n) // b)


@pytest.mark.parametrize("T,H,W,b,nc,qc,first,M", [
    (3, 3, 4, 2, 2, 1, 0, 18),
    (3, 3, 4, 2, 3, 2, 5, 31),
    (2, 4, 3, 4, 3, 1, 0, 18),        # W < H is fine for a raster order
    (2, 3, 3, 3, 3, 2, 2, 10),
])
def test_thw_neighbours_match_token_pair_brute_force(T, H, W, b, nc, qc, first, M):
    got = gilbert.neighbour_blocks(T, H, W, nc, b, qc, first, M, layout="thw")
    block = np.arange(nc * T * H * W) // b
    assert got == _brute_neighbours(T, H, W, nc, b, qc, first, M, block=block)


def _same_block_fraction(B):
    H, W = B.shape
    pairs = same = 0
    for y in range(H):
        for x in range(W):
            for dy in (-1, 0, 1):
                for dx in (-1, 0, 1):
                    y2, x2 = y + dy, x + dx
                    if (dy or dx) and 0 <= y2 < H and 0 <= x2 < W:
                        pairs += 1
                        same += int(B[y, x] == B[y2, x2])
    return same / pairs


def test_gilbert_keeps_adjacent_tokens_in_one_block_more_often_than_thw():
    # the pages' point of the Gilbert order: adjacent tokens stay adjacent, so
    # blocks are compact.  On the chunk-48 frame (32 x 48, 128-token blocks)
    # more in-frame 8-neighbour token pairs share a block under the Gilbert
    # order (0.878) than under THW-linear strips of 2.67 rows (0.734).
    T, H, W, b = 1, 32, 48, 128
    _, _, bg = gilbert.global_order(T, H, W, 1, b)
    _, _, bt = gilbert.thw_linear_order(T, H, W, 1, b)
    fg = _same_block_fraction(bg.reshape(H, W))
    ft = _same_block_fraction(bt.reshape(H, W))
    assert fg > ft + 0.1


@pytest.mark.parametrize("T,H,W", [(3, 3, 4), (4, 4, 8), (2, 32, 48)])
def test_first_frame_is_the_plain_curve_and_odd_frames_its_mirror(T, H, W):
    # mirror *alternate* frames starting from the plain map: frame 0 is the
    # frame curve itself (from cell (0, 0) to (W-1, 0)), frame 1 its mirror
    rank, cell, _ = gilbert.global_order(T, H, W, 2, 1)
    r = rank.reshape(2 * T, H, W)
    r2 = gilbert.frame_rank_map(W, H)
    assert np.array_equal(r[0], r2)
    assert np.array_equal(r[1] - H * W, r2[:, ::-1])
    assert int(cell[0]) == 0 and r[0][0, W - 1] == H * W - 1
    assert r[1][0, W - 1] == H * W and r[1][0, 0] == 2 * H * W - 1
