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

The inside/outside decisions turn floats into counts, so they are taken in
fp32 with the same operation order as the CUDA kernel (every product and sum
rounded separately, in the order written here); the ratios are fp64.
"""

from __future__ import annotations

import numpy as np

F = np.float32


def _f(x):
    return np.asarray(x, dtype=np.float32)


def obb(cam: np.ndarray, slab: np.ndarray):
    """Centre (3,), axes R (3x3, columns) and half extents (3,) of a slab.

    cam: [fx, fy, cx, cy, R00..R22 (row-major), Cx, Cy, Cz] (16 fp32)
    slab: [u0, u1, v0, v1, zlo, zhi] (fp32)
    """
    cam, slab = _f(cam), _f(slab)
    fx, fy, cx, cy = cam[0], cam[1], cam[2], cam[3]
    R = cam[4:13].reshape(3, 3)
    C = cam[13:16]
    u0, u1, v0, v1, zlo, zhi = slab[:6]
    zm = F(0.5) * F(zlo + zhi)
    um = F(0.5) * F(u0 + u1)
    vm = F(0.5) * F(v0 + v1)
    xl = F(F(F(um - cx) / fx) * zm)
    yl = F(F(F(vm - cy) / fy) * zm)
    centre = _cam_to_world(R, C, np.array([xl, yl, zm], dtype=F))
    half = np.array([F(F(F(F(u1 - u0) * F(0.5)) / fx) * zm),
                     F(F(F(F(v1 - v0) * F(0.5)) / fy) * zm),
                     F(F(0.5) * F(zhi - zlo))], dtype=F)
    return centre, R, half


def _cam_to_world(R, C, x):
    """C + R x with the kernel's rounding order: ((R0 x0 + R1 x1) + R2 x2) + C."""
    out = np.empty(3, dtype=F)
    for k in range(3):
        acc = F(R[k, 0] * x[0])
        acc = F(acc + F(R[k, 1] * x[1]))
        acc = F(acc + F(R[k, 2] * x[2]))
        out[k] = F(acc + C[k])
    return out


def _world_to_box(R, centre, X):
    """R^T (X - centre), same rounding order."""
    dx = np.array([F(X[0] - centre[0]), F(X[1] - centre[1]), F(X[2] - centre[2])], dtype=F)
    out = np.empty(3, dtype=F)
    for k in range(3):
        acc = F(R[0, k] * dx[0])
        acc = F(acc + F(R[1, k] * dx[1]))
        acc = F(acc + F(R[2, k] * dx[2]))
        out[k] = acc
    return out


def slab_iou(cam_i, slab_i, cam_r, slab_r, valid_r: bool, grid: int) -> float:
    """g for one (query slab, history slab) pair."""
    if not valid_r:
        return 0.0
    ci, Ri, hi = obb(cam_i, slab_i)
    cr, Rr, hr = obb(cam_r, slab_r)
    G = grid
    s = [F(F(F(2 * a + 1) / F(G)) - F(1.0)) for a in range(G)]
    n_in = 0
    for a in range(G):
        for b in range(G):
            for c in range(G):
                p = np.array([F(s[a] * hi[0]), F(s[b] * hi[1]), F(s[c] * hi[2])], dtype=F)
                X = _cam_to_world(Ri, ci, p)
                d = _world_to_box(Rr, cr, X)
                if abs(d[0]) <= hr[0] and abs(d[1]) <= hr[1] and abs(d[2]) <= hr[2]:
                    n_in += 1
    vi = 8.0 * float(hi[0]) * float(hi[1]) * float(hi[2])
    vr = 8.0 * float(hr[0]) * float(hr[1]) * float(hr[2])
    inter = vi * n_in / float(G ** 3)
    union = vi + vr - inter
    return inter / union if union > 0.0 else 0.0


def overlap(cams, q_cam, q_slab, h_cam, h_slab, h_valid, grid: int) -> np.ndarray:
    """g [N][M] for all query slabs against all history slabs."""
    N, M = len(q_cam), len(h_cam)
    g = np.zeros((N, M))
    for i in range(N):
        for r in range(M):
            g[i, r] = slab_iou(cams[q_cam[i]], q_slab[i], cams[h_cam[r]], h_slab[r],
                               bool(h_valid[r]), grid)
    return g


def _project(cam, X):
    """(u, v, z) of world point X in camera `cam`, kernel rounding order."""
    cam = _f(cam)
    fx, fy, cx, cy = cam[0], cam[1], cam[2], cam[3]
    R = cam[4:13].reshape(3, 3)
    x = _world_to_box(R, cam[13:16], X)  # camera frame: R^T (X - C)
    z = x[2]
    u = F(F(F(x[0] / z) * fx) + cx)
    v = F(F(F(x[1] / z) * fy) + cy)
    return u, v, z


def token_inside(cam_t, u, v, z, cam_r, slab_r) -> bool:
    """Does token (u, v) at depth z of camera cam_t fall inside slab r?"""
    if not z > 0:
        return False
    cam_t = _f(cam_t)
    fx, fy, cx, cy = cam_t[0], cam_t[1], cam_t[2], cam_t[3]
    R = cam_t[4:13].reshape(3, 3)
    xl = F(F(F(F(u) - cx) / fx) * F(z))
    yl = F(F(F(F(v) - cy) / fy) * F(z))
    X = _cam_to_world(R, cam_t[13:16], np.array([xl, yl, F(z)], dtype=F))
    pu, pv, pz = _project(cam_r, X)
    s = _f(slab_r)
    return bool(pz > 0 and s[0] <= pu < s[1] and s[2] <= pv < s[3] and s[4] <= pz <= s[5])


def coverage(cams, q_cam, q_uvz, h_cam, h_slab, h_valid, eta: float = 0.9):
    """rho [N] (fraction of covered tokens) and covered [N] (rho >= eta).

    q_uvz: [N][b][3] token coordinates and warped depth of each query block.
    """
    N, b = q_uvz.shape[0], q_uvz.shape[1]
    rho = np.zeros(N)
    for i in range(N):
        n_cov = 0
        for t in range(b):
            u, v, z = q_uvz[i, t]
            for r in range(len(h_cam)):
                if h_valid[r] and token_inside(cams[q_cam[i]], u, v, z, cams[h_cam[r]], h_slab[r]):
                    n_cov += 1
                    break
        rho[i] = n_cov / b
    return rho, (rho >= float(np.float32(eta))).astype(np.uint8)
