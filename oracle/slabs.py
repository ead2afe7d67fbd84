"""Slab-table build and recency-priority multiwarp (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages state (digest of arXiv 2610.22311, "Method steps", steps one
and two, Eq. 4-6, and "Prerequisites" (frustum slab); project page, "02 ·
Method", steps 01-02; onedev.kr summary, "How it differs"):

* after a chunk is decoded, the reconstruction backend gives depth,
  confidence, a mask and the pose; the reliable depth is back-projected and
  bucketed by Gilbert block, and every history KV block gets a frustum slab:
  its token rectangle plus the 10th / 90th percentile depth interval (Eq. 5);
* the current noisy chunk has no depth of its own: the first and last frame
  depths of the K = 30 most recent reconstructed chunks are forward-warped to
  the target camera, and each token takes the median of the newest frame
  that gives it at least k_warp = 2 samples (Eq. 6).

Readings taken where the pages are open:

* depth maps are given at s x s samples per latent token (s >= 1); sample
  (px, py) belongs to token (px // s, py // s) and sits at token coordinates
  ((px + 0.5) / s, (py + 0.5) / s);
* a sample is reliable when its mask is set, its confidence is >= c_min and
  its depth is > 0;
* a block's rectangle is the bounding box of its tokens in its frame:
  [min x, max x + 1) x [min y, max y + 1); its camera is its frame's; a block
  with fewer than n_min reliable samples gets an invalid slab (zeros);
* percentile q of n sorted values: linear interpolation between order
  statistics at h = (n - 1) q (numpy's default definition), in fp64 from the
  fp32 samples, rounded to fp32;
* a warped sample lands in target token (floor(u'), floor(v')) when its
  target depth is > 0 and 0 <= u' < W, 0 <= v' < H; its value is the target
  camera depth; the warp takes every source sample with depth > 0;
* the median of an even count is the mean of the two middle values (fp64,
  rounded to fp32); a token that no source frame gives k_warp samples stays a
  hole (depth 0);
* blocks never straddle frames (H W is a multiple of the block size).

The projections are plain fp64 arithmetic from the fp32 inputs (the
formulas of ``oracle.geometry``).  The target token of a sample is an integer
decided by floats: a sample whose projected position lies within the
marginal distance of a token edge (EPS_REL of ``oracle.geometry``, in world
units) could land in either neighbour in another precision, so the multiwarp
also reports the target tokens that such a sample touches ("unsure" tokens,
whose count, source and median are not fixed by the fp64 decision).
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Sequence

import numpy as np

from .geometry import EPS_REL, _cam, token_world

F = np.float32


def percentile_sorted(v: Sequence[float], q: float) -> float:
    """Linear interpolation between the order statistics of sorted v at (n-1) q."""
    n = len(v)
    h = (n - 1) * q
    lo = math.floor(h)
    t = h - lo
    if lo + 1 < n:
        a, b = float(v[lo]), float(v[lo + 1])
        return a + (b - a) * t
    return float(v[lo])


@dataclass
class SlabParams:
    s: int = 1            # depth samples per token along each axis
    c_min: float = 0.5    # minimum confidence of a reliable sample
    n_min: int = 8        # minimum reliable samples of a valid slab
    p_lo: float = 0.10
    p_hi: float = 0.90


def slab_table(depth, conf, mask, cell_of_rank, H: int, W: int, b: int, frame_base: int,
               first_block: int, n_blocks: int, prm: SlabParams):
    """Frustum slabs of blocks first_block .. first_block + n_blocks - 1.

    depth, conf [F][H s][W s] fp32 and mask [F][H s][W s] uint8 hold global
    frames frame_base .. frame_base + F - 1; cell_of_rank maps a global rank
    to the cell index (f H + y) W + x (any block order).  Returns slab
    [n][6] fp32, cam [n] int32 (the global frame), valid [n] int32.
    """
    s = prm.s
    HW = H * W
    slab = np.zeros((n_blocks, 6), dtype=np.float32)
    cam = np.zeros(n_blocks, dtype=np.int32)
    valid = np.zeros(n_blocks, dtype=np.int32)
    for j in range(n_blocks):
        r = first_block + j
        cells = [int(cell_of_rank[r * b + t]) for t in range(b)]
        f = cells[0] // HW
        lf = f - frame_base
        xs = [(c % HW) % W for c in cells]
        ys = [(c % HW) // W for c in cells]
        cam[j] = f
        samples = []
        for x, y in zip(xs, ys):
            for py in range(y * s, y * s + s):
                for px in range(x * s, x * s + s):
                    z = float(depth[lf, py, px])
                    ok = mask is None or mask[lf, py, px] != 0
                    ok = ok and (conf is None or float(conf[lf, py, px]) >= float(F(prm.c_min)))
                    if ok and z > 0.0 and math.isfinite(z):
                        samples.append(z)
        if len(samples) < prm.n_min or not samples:
            continue
        samples.sort()
        slab[j] = [min(xs), max(xs) + 1, min(ys), max(ys) + 1,
                   F(percentile_sorted(samples, prm.p_lo)),
                   F(percentile_sorted(samples, prm.p_hi))]
        valid[j] = 1
    return slab, cam, valid


def block_tokens(depth, conf, mask, cell_of_rank, H: int, W: int, b: int, frame_base: int,
                 first_block: int, n_blocks: int, c_min: float = 0.5) -> np.ndarray:
    """[n][b][3]: the tokens of each block in rank order as (x + 0.5, y + 0.5,
    depth), depth 0 where it is not a reliable sample (s = 1): the per-token
    input of the coverage when depth is a multiwarp map."""
    HW = H * W
    out = np.zeros((n_blocks, b, 3), dtype=np.float32)
    for j in range(n_blocks):
        for t in range(b):
            c = int(cell_of_rank[(first_block + j) * b + t])
            f, rem = divmod(c, HW)
            y, x = divmod(rem, W)
            z = float(depth[f - frame_base, y, x])
            ok = z > 0.0 and math.isfinite(z) and (mask is None or mask[f - frame_base, y, x] != 0)
            ok = ok and (conf is None or float(conf[f - frame_base, y, x]) >= float(F(c_min)))
            out[j, t] = [x + 0.5, y + 0.5, z if ok else 0.0]
    return out


def warp_sample(cam_src, cam_tgt, u, v, z, H: int, W: int):
    """Warp source point (u, v) at depth z into the target camera.

    Returns (cell, depth, margin, candidates): cell = (x, y) of the target
    token it lands in, or None when it does not land in the frame (target
    depth <= 0 or outside [0, W) x [0, H)); depth = the target-camera depth;
    margin = the distance in world units to the nearest token edge (frame
    edges included) or to the camera plane; candidates = the in-frame cells
    the point lies in or touches within the marginal distance.
    """
    X = token_world(cam_src, u, v, z)
    fx, fy, cx, cy, R, C = _cam(cam_tgt)
    d = R.T @ (X - C)
    pz = float(d[2])
    eps = EPS_REL * max(1.0, float(np.abs(X).max()), float(np.abs(C).max()))
    if not pz > 0.0:
        return None, pz, -pz, []
    pu = d[0] / pz * fx + cx
    pv = d[1] / pz * fy + cy
    mu = abs(pu - round(pu)) * pz / fx
    mv = abs(pv - round(pv)) * pz / fy
    margin = min(mu, mv, pz)
    du, dv = eps * fx / pz, eps * fy / pz          # the marginal distance in token units
    xs = {math.floor(pu - du), math.floor(pu), math.floor(pu + du)}
    ys = {math.floor(pv - dv), math.floor(pv), math.floor(pv + dv)}
    cand = [(x, y) for x in xs for y in ys if 0 <= x < W and 0 <= y < H]
    if not (0.0 <= pu < W and 0.0 <= pv < H):
        return None, pz, margin, cand
    return (math.floor(pu), math.floor(pv)), pz, margin, cand


def multiwarp_bounds(cams, src_depth, src_cam: Sequence[int], tgt_cam: int, H: int, W: int,
                     s: int, k_warp: int = 2):
    """z^Q [H][W] of the target camera from source depths [S][H s][W s]
    (src_cam[k] is the camera of source k, newest first), and the [H][W]
    mask of unsure tokens (touched by a sample whose landing is marginal)."""
    S = len(src_cam)
    per_src: List[dict] = []
    unsure = np.zeros((H, W), dtype=bool)
    for k in range(S):
        got: dict = {}
        dk = src_depth[k]
        cam_s, cam_t = cams[src_cam[k]], cams[tgt_cam]
        for py in range(H * s):
            for px in range(W * s):
                z = float(dk[py, px])
                if not z > 0.0:
                    continue
                u = (px + 0.5) / s
                v = (py + 0.5) / s
                cell, depth, margin, cand = warp_sample(cam_s, cam_t, u, v, z, H, W)
                eps = EPS_REL * max(1.0, float(np.abs(token_world(cam_s, u, v, z)).max()),
                                    float(np.abs(np.asarray(cam_t, np.float64)[13:16]).max()))
                if margin <= eps:
                    for (x, y) in cand:
                        unsure[y, x] = True
                if cell is not None:
                    got.setdefault(cell, []).append(depth)
        per_src.append(got)
    zq = np.zeros((H, W), dtype=np.float32)
    for y in range(H):
        for x in range(W):
            for got in per_src:
                vals = got.get((x, y), [])
                if len(vals) >= k_warp:
                    zq[y, x] = np.float32(np.median(np.asarray(vals, dtype=np.float64)))
                    break
    return zq, unsure


def multiwarp(cams, src_depth, src_cam: Sequence[int], tgt_cam: int, H: int, W: int, s: int,
              k_warp: int = 2) -> np.ndarray:
    """z^Q [H][W] of the target camera (see multiwarp_bounds)."""
    return multiwarp_bounds(cams, src_depth, src_cam, tgt_cam, H, W, s, k_warp)[0]
