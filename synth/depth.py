"""Seeded synthetic depth maps of a static room seen from a moving camera.

Input draws for the slab-table build and the multiwarp: per-frame depth,
confidence and mask at s x s samples per latent token, in the camera
convention of the geometry calls (pinhole in token units, R world-from-camera
row-major, camera z forward, y down).  The scene is a box-shaped room (floor,
ceiling, side walls, back wall) with a few axis-aligned boxes standing on the
floor; depth is the camera-z distance of the first surface hit by the ray of
each sample.  This is how the inputs are made, not part of the method: the
method only consumes depth, it never casts rays.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class Rollout:
    cams: np.ndarray    # [F][16] float32
    depth: np.ndarray   # [F][H s][W s] float32 (0 where nothing was hit)
    conf: np.ndarray    # [F][H s][W s] float32 in [0, 1]
    mask: np.ndarray    # [F][H s][W s] uint8


def _yaw(a: float) -> np.ndarray:
    c, s = np.cos(a), np.sin(a)
    return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])


def make_rollout(seed: int, n_frames: int, H: int, W: int, s: int = 1,
                 step: float = 0.02, p_unreliable: float = 0.1) -> Rollout:
    """n_frames frames of H x W tokens (s x s samples each).

    The camera starts at z = -2 facing +z, advances `step` per frame with a
    slow sideways sway and yaw; the room spans x in [-5, 5], y in [-2.5, 1.2]
    (floor at y = 1.2, image y points down) and z up to 14.  Confidence is
    U[0, 1] with a fraction `p_unreliable` of the samples below 0.2; the mask
    drops 3 % of the samples.
    """
    rng = np.random.default_rng(seed)
    n_box = 4
    bx = rng.uniform(-3.5, 3.5, n_box)
    bz = rng.uniform(3.0, 11.0, n_box)
    bw = rng.uniform(0.4, 1.2, n_box)
    bh = rng.uniform(0.5, 2.0, n_box)
    lo = np.stack([bx - bw, 1.2 - bh, bz - bw], 1)
    hi = np.stack([bx + bw, np.full(n_box, 1.2), bz + bw], 1)

    f = 0.75 * W
    cams = np.zeros((n_frames, 16), dtype=np.float32)
    Hs, Ws = H * s, W * s
    depth = np.zeros((n_frames, Hs, Ws), dtype=np.float32)
    py, px = np.meshgrid(np.arange(Hs), np.arange(Ws), indexing="ij")
    u = (px + 0.5) / s
    v = (py + 0.5) / s
    for k in range(n_frames):
        R = _yaw(0.15 * np.sin(0.02 * k))
        C = np.array([0.8 * np.sin(0.015 * k), 0.0, -2.0 + step * k])
        cams[k] = [f, f, W / 2.0, H / 2.0, *R.reshape(-1), *C]
        d_cam = np.stack([(u - W / 2.0) / f, (v - H / 2.0) / f, np.ones_like(u)], -1)
        d = d_cam @ R.T                      # world directions, camera-z component 1
        t = np.full(u.shape, np.inf)
        with np.errstate(divide="ignore", invalid="ignore"):
            for axis, planes in ((0, (-5.0, 5.0)), (1, (-2.5, 1.2)), (2, (14.0,))):
                for p in planes:
                    tt = (p - C[axis]) / d[..., axis]
                    t = np.where((tt > 1e-6) & (tt < t), tt, t)
            for j in range(n_box):
                t0 = (lo[j] - C) / d
                t1 = (hi[j] - C) / d
                tn = np.nanmax(np.minimum(t0, t1), axis=-1)
                tf = np.nanmin(np.maximum(t0, t1), axis=-1)
                hit = (tn <= tf) & (tn > 1e-6)
                t = np.where(hit & (tn < t), tn, t)
        depth[k] = np.where(np.isfinite(t), t, 0.0).astype(np.float32)
    conf = rng.random(depth.shape).astype(np.float32)
    low = rng.random(depth.shape) < p_unreliable
    conf[low] = (0.2 * rng.random(int(low.sum()))).astype(np.float32)
    conf[~low] = np.maximum(conf[~low], np.float32(0.2))
    mask = (rng.random(depth.shape) >= 0.03).astype(np.uint8)
    return Rollout(cams, depth, conf, mask)
