"""Global-aligned Gilbert order and 26-neighbour safeguard blocks (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix (Velox project page, "02 · Method", "Keeping neighbours
adjacent in the block order", figure "Incremental Gilbert order"; arXiv
2610.22311 digest, "Prerequisites", "Gilbert space-filling curve"):

* a Gilbert (generalised Hilbert) space-filling curve meanders over the 2-D
  latent grid so that neighbouring tokens get nearby sequence ranks;
* the single-chunk rank map is built once and concatenated chunk after chunk;
  a plain repeat breaks temporal adjacency at the chunk seam, and mirroring the
  mapping horizontally on alternate chunks restores it (toy case: 3 frames per
  chunk, latent 3 x 4, block size 2);
* the order is the KV storage layout, the id space of 128-token blocks and the
  domain of the 26-neighbour safeguard.

Reading taken where the pages leave the construction open: each frame is
walked by the 2-D Gilbert curve from cell (0, 0) to cell (W-1, 0); the curve is
mirrored in x on every frame of odd *global* frame index, so consecutive frames
join with a unit step in t.  With an odd number of frames per chunk this is
exactly "mirror alternate chunks"; with an even number it keeps the seams
adjacent where a literal per-chunk mirror would break them.  Halving in the
curve construction rounds toward minus infinity (floor division).  Supported
frames have W >= H and are not (W odd, H even), the case in which no unit-step
path from (0, 0) to (W-1, 0) exists.

Pins (tests/test_oracle_gilbert.py): a bijection with unit steps across every
block, frame and chunk seam; contiguous chunks; the mirror rule; and, on
2^k x 2^k frames, the textbook Hilbert curve cell for cell.  On other frame
shapes (the 32 x 48 latent frame among them), which unit-step path the
construction picks is fixed only by those invariants.  Against the authors'
own figures it is parity unpinned: the figures' ranks are not in the text.
"""

from __future__ import annotations

import numpy as np


def _sign(v: int) -> int:
    return (v > 0) - (v < 0)


def frame_curve(width: int, height: int) -> list:
    """Cells (x, y) of a width x height frame in 2-D Gilbert visit order.

    The generalised Hilbert construction for arbitrary rectangles (J. Cerveny,
    "gilbert", 2019) restated: a rectangle is given by a start corner, a major
    edge vector and a minor edge vector; the path starts in the corner cell
    and ends in the last cell along the major edge on the same side.  Long
    rectangles (2 * major > 3 * minor) are cut across the major edge into two
    halves walked one after the other; others are cut into three: a piece
    covering the near half of the minor edge with the two edges swapped, the
    full-length remainder, and a mirrored piece that returns along the far
    side.  Halves are made even when the edge is longer than 2 cells.
    """
    if width < 1 or height < 1:
        raise ValueError("empty frame")
    if width < height:
        raise ValueError("frames with W < H are not supported")
    cells: list = []
    _walk(cells, 0, 0, width, 0, 0, height)
    return cells


def _walk(cells, x, y, ax, ay, bx, by):
    # The steps below are those of Jakub Cerveny's published generalised
    # Hilbert ("gilbert") construction, which this function restates; that
    # project is distributed under the BSD 2-Clause licence, whose notice is
    # reproduced here:
    #
    #   Copyright (c) 2018, Jakub Cerveny.  All rights reserved.
    #   Redistribution and use in source and binary forms, with or without
    #   modification, are permitted provided that the following conditions
    #   are met: 1. Redistributions of source code must retain the above
    #   copyright notice, this list of conditions and the following
    #   disclaimer.  2. Redistributions in binary form must reproduce the
    #   above copyright notice, this list of conditions and the following
    #   disclaimer in the documentation and/or other materials provided with
    #   the distribution.
    #   THIS SOFTWARE IS PROVIDED BY THE COPYRIGHT HOLDERS AND CONTRIBUTORS
    #   "AS IS" AND ANY EXPRESS OR IMPLIED WARRANTIES, INCLUDING, BUT NOT
    #   LIMITED TO, THE IMPLIED WARRANTIES OF MERCHANTABILITY AND FITNESS FOR
    #   A PARTICULAR PURPOSE ARE DISCLAIMED.  IN NO EVENT SHALL THE COPYRIGHT
    #   HOLDER OR CONTRIBUTORS BE LIABLE FOR ANY DIRECT, INDIRECT, INCIDENTAL,
    #   SPECIAL, EXEMPLARY, OR CONSEQUENTIAL DAMAGES (INCLUDING, BUT NOT
    #   LIMITED TO, PROCUREMENT OF SUBSTITUTE GOODS OR SERVICES; LOSS OF USE,
    #   DATA, OR PROFITS; OR BUSINESS INTERRUPTION) HOWEVER CAUSED AND ON ANY
    #   THEORY OF LIABILITY, WHETHER IN CONTRACT, STRICT LIABILITY, OR TORT
    #   (INCLUDING NEGLIGENCE OR OTHERWISE) ARISING IN ANY WAY OUT OF THE USE
    #   OF THIS SOFTWARE, EVEN IF ADVISED OF THE POSSIBILITY OF SUCH DAMAGE.
    n_major = abs(ax + ay)
    n_minor = abs(bx + by)
    ux, uy = _sign(ax), _sign(ay)   # unit step along the major edge
    vx, vy = _sign(bx), _sign(by)   # unit step along the minor edge
    if n_minor == 1:                # a single line along the major edge
        for k in range(n_major):
            cells.append((x + k * ux, y + k * uy))
        return
    if n_major == 1:                # a single line along the minor edge
        for k in range(n_minor):
            cells.append((x + k * vx, y + k * vy))
        return
    hax, hay = ax // 2, ay // 2     # floor halves of both edges
    hbx, hby = bx // 2, by // 2
    if 2 * n_major > 3 * n_minor:
        if abs(hax + hay) % 2 == 1 and n_major > 2:
            hax, hay = hax + ux, hay + uy
        _walk(cells, x, y, hax, hay, bx, by)
        _walk(cells, x + hax, y + hay, ax - hax, ay - hay, bx, by)
    else:
        if abs(hbx + hby) % 2 == 1 and n_minor > 2:
            hbx, hby = hbx + vx, hby + vy
        _walk(cells, x, y, hbx, hby, hax, hay)
        _walk(cells, x + hbx, y + hby, ax, ay, bx - hbx, by - hby)
        _walk(cells, x + (ax - ux) + (hbx - vx), y + (ay - uy) + (hby - vy),
              -hbx, -hby, -(ax - hax), -(ay - hay))


def frame_rank_map(width: int, height: int) -> np.ndarray:
    """r2[y, x] = position of cell (x, y) on the frame curve."""
    r2 = np.full((height, width), -1, dtype=np.int64)
    for k, (x, y) in enumerate(frame_curve(width, height)):
        r2[y, x] = k
    return r2


def check_supported(T: int, H: int, W: int, b: int) -> None:
    if min(T, H, W, b) < 1:
        raise ValueError("non-positive lattice size")
    if W < H:
        raise ValueError("W < H unsupported")
    if W % 2 == 1 and H % 2 == 0:
        raise ValueError("W odd with H even has no unit-step frame path")
    if (T * H * W) % b != 0:
        raise ValueError("T*H*W must be a multiple of the block size")


def global_order(T: int, H: int, W: int, n_chunks: int, b: int):
    """Global Gilbert order over n_chunks chunks of T frames of H x W cells.

    Cell index c = (f * H + y) * W + x with global frame f = chunk * T + t.
    Returns (rank_of_cell, cell_of_rank, block_of_cell), all int64 arrays of
    n_chunks * T * H * W entries; block = rank // b.
    """
    check_supported(T, H, W, b)
    r2 = frame_rank_map(W, H)
    F = n_chunks * T
    HW = H * W
    rank = np.empty((F, H, W), dtype=np.int64)
    for f in range(F):
        frame = r2[:, ::-1] if f % 2 == 1 else r2
        rank[f] = f * HW + frame
    rank_of_cell = rank.reshape(-1)
    cell_of_rank = np.empty_like(rank_of_cell)
    cell_of_rank[rank_of_cell] = np.arange(rank_of_cell.size)
    return rank_of_cell, cell_of_rank, rank_of_cell // b


def thw_linear_order(T: int, H: int, W: int, n_chunks: int, b: int):
    """The THW-linear order the pages compare against (project page, figure
    "THW-linear against global Gilbert order"): tokens flattened frame by
    frame, each frame row by row, rank(f, y, x) = (f * H + y) * W + x.
    Same return convention as global_order."""
    if min(T, H, W, b) < 1:
        raise ValueError("non-positive lattice size")
    if (T * H * W) % b != 0:
        raise ValueError("T*H*W must be a multiple of the block size")
    F = n_chunks * T
    rank = np.empty((F, H, W), dtype=np.int64)
    for f in range(F):
        for y in range(H):
            for x in range(W):
                rank[f, y, x] = (f * H + y) * W + x
    rank_of_cell = rank.reshape(-1)
    cell_of_rank = np.empty_like(rank_of_cell)
    cell_of_rank[rank_of_cell] = np.arange(rank_of_cell.size)
    return rank_of_cell, cell_of_rank, rank_of_cell // b


def neighbour_blocks(T: int, H: int, W: int, n_chunks: int, b: int,
                     q_chunk: int, cache_first_block: int, n_cache_blocks: int,
                     layout: str = "gilbert"):
    """26-neighbour safeguard blocks of every query block of chunk q_chunk.

    Reading of "Gilbert 26-neighbour blocks" (digest, "Method steps", Eq. 14;
    onedev.kr summary, "How it differs"): history block u is a safeguard of
    query block i when u != i and some token of u lies in the 3 x 3 x 3 lattice
    neighbourhood (global frame, y, x; no wrap) of some token of i.  Only
    blocks inside the cache range are kept, as cache ids
    (global block id - cache_first_block), ascending.

    layout "gilbert" (the global Gilbert order) or "thw" (THW-linear).
    Returns a list (one entry per query block of the chunk) of int lists.
    """
    order = {"gilbert": global_order, "thw": thw_linear_order}[layout]
    _, _, block_of_cell = order(T, H, W, n_chunks, b)
    F = n_chunks * T
    blk = block_of_cell.reshape(F, H, W)
    per_chunk = T * H * W // b
    lo, hi = cache_first_block, cache_first_block + n_cache_blocks
    out = []
    for i in range(per_chunk):
        qb = q_chunk * per_chunk + i
        fs, ys, xs = np.nonzero(blk == qb)
        found = set()
        for f, y, x in zip(fs, ys, xs):
            for df in (-1, 0, 1):
                for dy in (-1, 0, 1):
                    for dx in (-1, 0, 1):
                        if df == 0 and dy == 0 and dx == 0:
                            continue
                        f2, y2, x2 = f + df, y + dy, x + dx
                        if 0 <= f2 < F and 0 <= y2 < H and 0 <= x2 < W:
                            u = int(blk[f2, y2, x2])
                            if u != qb and lo <= u < hi:
                                found.add(u - lo)
        out.append(sorted(found))
    return out
