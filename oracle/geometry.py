"""Frustum-slab overlap g_{i,r} and coverage rho_i (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages state (Velox project page, "02 · Method", steps 01-02 and the
glossary entry for g; digest of arXiv 2610.22311, "Prerequisites" (frustum
slab and OBB overlap) and "Method steps", steps one to three, Eq. 7-8;
onedev.kr summary, "How it differs"):

* every historical KV block is summarised as a frustum slab: a token
  rectangle in its source camera plus a robust depth interval [z-, z+];
* the query block gets a depth interval of its own from the warped depth;
* g_{i,r} is the overlap (intersection over union) of the two slabs in
  world space, each approximated by a camera-facing oriented box (OBB), with
  the intersection volume approximated on a grid;
* rho_i is the fraction of the query block's tokens whose (warped) depth
  falls inside a valid past slab; the block is covered when rho_i >= 0.9.

Readings taken where the pages are open:

* pinhole cameras in latent-token units: pixel (u, v) at depth z is the
  camera-frame point ((u - cx) / fx * z, (v - cy) / fy * z, z); the world
  point is C + R x (R world-from-camera, C the camera centre);
* the OBB of a slab has the camera's axes, its centre on the ray through the
  rectangle centre at the mid depth zm = (z- + z+)/2, half extents
  (u1 - u0)/(2 fx) zm, (v1 - v0)/(2 fy) zm and (z+ - z-)/2;
* the intersection is estimated on the G x G x G cell centres of the query
  OBB: inter = vol_i * (inside count) / G^3, IoU = inter / (vol_i + vol_r -
  inter); an invalid slab gives 0;
* a token "falls inside" slab r when its world point, projected into slab
  r's camera, lands in the rectangle [u0, u1) x [v0, v1) at a depth in
  [z-, z+]; a token with depth <= 0 (a hole) is never covered.

Everything here is plain fp64 arithmetic from the fp32 inputs (numpy matrix
products, no imposed operation order).  The inside/outside decisions turn
floats into counts, and an implementation in another precision may decide a
point that lies within rounding distance of a face the other way.  So every
decision also yields its distance to the deciding face, in world units; a
decision closer than EPS_REL x (the size of the coordinates involved) is
"marginal".  The *_bounds functions return, next to the value, the values
that every choice of the marginal decisions can give: a count in
[n_lo, n_hi] and the matching g or rho interval.
"""

from __future__ import annotations

import numpy as np

# Relative size of a marginal decision.  An fp32 evaluation of these
# formulas (about 20 roundings of coordinates of size s) lands within a few
# 1e-6 s of the fp64 value; 1e-5 s leaves a margin of several times that.
EPS_REL = 1e-5


def _cam(cam):
    c = np.asarray(cam, dtype=np.float64)
    return c[0], c[1], c[2], c[3], c[4:13].reshape(3, 3), c[13:16]


def obb(cam: np.ndarray, slab: np.ndarray):
    """Centre (3,), axes R (3x3, columns) and half extents (3,) of a slab, fp64.

    cam: [fx, fy, cx, cy, R00..R22 (row-major), Cx, Cy, Cz] (16 fp32)
    slab: [u0, u1, v0, v1, zlo, zhi] (fp32)
    """
    fx, fy, cx, cy, R, C = _cam(cam)
    u0, u1, v0, v1, zlo, zhi = np.asarray(slab, dtype=np.float64)[:6]
    zm = 0.5 * (zlo + zhi)
    local = np.array([(0.5 * (u0 + u1) - cx) / fx * zm, (0.5 * (v0 + v1) - cy) / fy * zm, zm])
    centre = C + R @ local
    half = np.array([(u1 - u0) / (2.0 * fx) * zm, (v1 - v0) / (2.0 * fy) * zm,
                     0.5 * (zhi - zlo)])
    return centre, R, half


def _grid_points(ci, Ri, hi, G):
    """World positions of the G^3 cell centres of a box: [G^3][3] (a, b, c order)."""
    s = (2.0 * np.arange(G) + 1.0) / G - 1.0
    a, b, c = np.meshgrid(s, s, s, indexing="ij")
    local = np.stack([a.ravel() * hi[0], b.ravel() * hi[1], c.ravel() * hi[2]], axis=1)
    return ci + local @ Ri.T


def slab_iou_counts(cam_i, slab_i, cam_r, slab_r, valid_r: bool, grid: int):
    """(n_in, n_lo, n_hi, vol_i, vol_r) of one (query, history) slab pair.

    n_in counts the query box's grid points inside the history box; n_lo
    those inside by more than the marginal distance, n_hi those inside or
    outside by less than it.  An invalid history slab gives all zeros.
    """
    G = grid
    if not valid_r:
        return 0, 0, 0, 0.0, 0.0
    ci, Ri, hi = obb(cam_i, slab_i)
    cr, Rr, hr = obb(cam_r, slab_r)
    X = _grid_points(ci, Ri, hi, G)
    d = (X - cr) @ Rr                      # box-frame coordinates R_r^T (X - c_r)
    margin = np.min(hr[None, :] - np.abs(d), axis=1)   # > 0 inside, < 0 outside
    scale = max(1.0, float(np.abs(X).max()), float(np.abs(cr).max()), float(hr.max()))
    eps = EPS_REL * scale
    n_in = int(np.count_nonzero(margin >= 0.0))
    n_lo = int(np.count_nonzero(margin > eps))
    n_hi = int(np.count_nonzero(margin >= -eps))
    vi = 8.0 * hi[0] * hi[1] * hi[2]
    vr = 8.0 * hr[0] * hr[1] * hr[2]
    return n_in, n_lo, n_hi, vi, vr


def iou_from_count(n: int, vi: float, vr: float, grid: int) -> float:
    """IoU for an inside count n: inter = vi n / G^3, g = inter / (vi + vr - inter)."""
    inter = vi * n / float(grid ** 3)
    union = vi + vr - inter
    return inter / union if union > 0.0 else 0.0


def slab_iou(cam_i, slab_i, cam_r, slab_r, valid_r: bool, grid: int) -> float:
    """g for one (query slab, history slab) pair."""
    n, _, _, vi, vr = slab_iou_counts(cam_i, slab_i, cam_r, slab_r, valid_r, grid)
    return iou_from_count(n, vi, vr, grid) if valid_r else 0.0


def overlap_bounds(cams, q_cam, q_slab, h_cam, h_slab, h_valid, grid: int):
    """g, g_lo, g_hi [N][M]: the IoU and its range over the marginal decisions."""
    N, M = len(q_cam), len(h_cam)
    g = np.zeros((N, M))
    lo = np.zeros((N, M))
    hi = np.zeros((N, M))
    for i in range(N):
        for r in range(M):
            n, n_lo, n_hi, vi, vr = slab_iou_counts(cams[q_cam[i]], q_slab[i], cams[h_cam[r]],
                                                    h_slab[r], bool(h_valid[r]), grid)
            if h_valid[r]:
                g[i, r] = iou_from_count(n, vi, vr, grid)
                lo[i, r] = iou_from_count(n_lo, vi, vr, grid)
                hi[i, r] = iou_from_count(n_hi, vi, vr, grid)
    return g, lo, hi


def overlap(cams, q_cam, q_slab, h_cam, h_slab, h_valid, grid: int) -> np.ndarray:
    """g [N][M] for all query slabs against all history slabs."""
    return overlap_bounds(cams, q_cam, q_slab, h_cam, h_slab, h_valid, grid)[0]


def token_world(cam_t, u, v, z) -> np.ndarray:
    """World point of token (u, v) at depth z of camera cam_t."""
    fx, fy, cx, cy, R, C = _cam(cam_t)
    u, v, z = float(u), float(v), float(z)
    return C + R @ np.array([(u - cx) / fx * z, (v - cy) / fy * z, z])


def inside_margin(X: np.ndarray, cam_r, slab_r):
    """(inside, margin) of world point X against slab r: inside when X
    projects into [u0, u1) x [v0, v1) at a depth in [z-, z+]; margin is the
    distance to the nearest face of that frustum piece in world units
    (image-plane distances times depth / focal length), as a lower bound of
    how far X can move before the decision changes."""
    fx, fy, cx, cy, R, C = _cam(cam_r)
    d = R.T @ (X - C)
    pz = d[2]
    if pz <= 0.0:
        return False, float(-pz)
    pu = d[0] / pz * fx + cx
    pv = d[1] / pz * fy + cy
    u0, u1, v0, v1, zlo, zhi = np.asarray(slab_r, dtype=np.float64)[:6]
    inside = (u0 <= pu < u1) and (v0 <= pv < v1) and (zlo <= pz <= zhi)
    du = min(abs(pu - u0), abs(u1 - pu)) * pz / fx
    dv = min(abs(pv - v0), abs(v1 - pv)) * pz / fy
    dz = min(abs(pz - zlo), abs(zhi - pz))
    if inside:
        margin = min(du, dv, dz)
    else:
        # outside: the distance to the nearest violated face bounds the move
        # needed to become inside from below by that face alone
        viol = []
        if not (u0 <= pu < u1):
            viol.append(du)
        if not (v0 <= pv < v1):
            viol.append(dv)
        if not (zlo <= pz <= zhi):
            viol.append(dz)
        margin = max(viol)
    return bool(inside), float(margin)


def token_inside(cam_t, u, v, z, cam_r, slab_r) -> bool:
    """Does token (u, v) at depth z of camera cam_t fall inside slab r?"""
    if not z > 0:
        return False
    return inside_margin(token_world(cam_t, u, v, z), cam_r, slab_r)[0]


def _inside_margin_many(X: np.ndarray, cams_r: np.ndarray, slabs_r: np.ndarray):
    """inside_margin of one world point against many slabs at once: the same
    formulas, one row per slab (cams_r [n][16], slabs_r [n][6])."""
    c = np.asarray(cams_r, dtype=np.float64)
    fx, fy, cx, cy = c[:, 0], c[:, 1], c[:, 2], c[:, 3]
    R = c[:, 4:13].reshape(-1, 3, 3)
    C = c[:, 13:16]
    d = np.einsum("nji,nj->ni", R, X[None, :] - C)   # R^T (X - C) per slab
    pz = d[:, 2]
    with np.errstate(divide="ignore", invalid="ignore"):
        pu = d[:, 0] / pz * fx + cx
        pv = d[:, 1] / pz * fy + cy
    sl = np.asarray(slabs_r, dtype=np.float64)
    u0, u1, v0, v1, zlo, zhi = (sl[:, k] for k in range(6))
    in_u = (u0 <= pu) & (pu < u1)
    in_v = (v0 <= pv) & (pv < v1)
    in_z = (zlo <= pz) & (pz <= zhi)
    front = pz > 0.0
    inside = front & in_u & in_v & in_z
    du = np.minimum(np.abs(pu - u0), np.abs(u1 - pu)) * pz / fx
    dv = np.minimum(np.abs(pv - v0), np.abs(v1 - pv)) * pz / fy
    dz = np.minimum(np.abs(pz - zlo), np.abs(zhi - pz))
    m_in = np.minimum(np.minimum(du, dv), dz)
    m_out = np.maximum(np.maximum(np.where(in_u, 0.0, du), np.where(in_v, 0.0, dv)),
                       np.where(in_z, 0.0, dz))
    margin = np.where(front, np.where(inside, m_in, m_out), -pz)
    return inside, margin


def coverage_bounds(cams, q_cam, q_uvz, h_cam, h_slab, h_valid):
    """Covered token counts n, n_lo, n_hi [N] of every query block.

    A token counts in n when some valid slab holds it; in n_lo when some
    valid slab holds it by more than the marginal distance; in n_hi when some
    valid slab holds it or misses it by less than the marginal distance.
    """
    N, b = q_uvz.shape[0], q_uvz.shape[1]
    n = np.zeros(N, dtype=np.int64)
    n_lo = np.zeros(N, dtype=np.int64)
    n_hi = np.zeros(N, dtype=np.int64)
    valid = np.flatnonzero(np.asarray(h_valid) != 0)
    cams = np.asarray(cams)
    cams_r = cams[np.asarray(h_cam)[valid]]
    slabs_r = np.asarray(h_slab)[valid]
    c_size = np.abs(cams_r[:, 13:16].astype(np.float64)).max(axis=1) if len(valid) else None
    for i in range(N):
        cam_t = cams[q_cam[i]]
        for t in range(b):
            u, v, z = (float(x) for x in q_uvz[i, t])
            if not z > 0 or len(valid) == 0:
                continue  # a hole is never covered
            X = token_world(cam_t, u, v, z)
            eps = EPS_REL * np.maximum(max(1.0, float(np.abs(X).max())), c_size)
            inside, margin = _inside_margin_many(X, cams_r, slabs_r)
            n[i] += bool(inside.any())
            n_lo[i] += bool((inside & (margin > eps)).any())
            n_hi[i] += bool((inside | (margin <= eps)).any())
    return n, n_lo, n_hi


def coverage(cams, q_cam, q_uvz, h_cam, h_slab, h_valid, eta: float = 0.9):
    """rho [N] (fraction of covered tokens) and covered [N] (rho >= eta).

    q_uvz: [N][b][3] token coordinates and warped depth of each query block.
    """
    b = q_uvz.shape[1]
    n, _, _ = coverage_bounds(cams, q_cam, q_uvz, h_cam, h_slab, h_valid)
    rho = n / b
    return rho, (rho >= float(np.float32(eta))).astype(np.uint8)
