"""Seeded synthetic camera paths, frustum slabs and warped query tokens.

Draws the inputs of the slab-overlap and coverage step with the structure the
Velox pages describe: a camera that moves through a static scene frame by
frame, every history KV block summarised by a token rectangle of its frame plus
a depth interval, and each query block's tokens carrying a warped depth with
holes (depth 0) where the warp found nothing.  It computes none of the
method's arithmetic (no projection, no box, no overlap, no coverage): cameras,
rectangles and depths are independent random draws.

Layouts (all fp32 unless stated):

* ``cams``   [n_cams][16]: fx, fy, cx, cy, R (world-from-camera, row-major),
  C (camera centre).
* ``*_slab`` [n][6]: u0, u1, v0, v1, zlo, zhi (token units, depth units).
* ``*_cam``  [n] int32 camera index; ``h_valid`` [n] int32 (0/1).
* ``q_uvz``  [N][b][3]: u, v, depth of every query token.
* ``pack_slabs`` turns (slab, cam, valid) into the [n][8] int32 records the
  C-ABI takes (six fp32 bit patterns, then cam, then valid).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class Scene:
    cams: np.ndarray
    q_slab: np.ndarray
    q_cam: np.ndarray
    q_uvz: np.ndarray
    h_slab: np.ndarray
    h_cam: np.ndarray
    h_valid: np.ndarray

    @property
    def n_cams(self) -> int:
        return self.cams.shape[0]


def _yaw(a: float) -> np.ndarray:
    c, s = np.cos(a), np.sin(a)
    return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])


def make_scene(seed: int, N: int, M: int, b: int = 128, frame_hw=(32, 48),
               block_hw=(8, 16), p_invalid: float = 0.1) -> Scene:
    """N query blocks (the frames after the history) and M history blocks.

    Blocks tile each frame row-major by ``block_hw`` token rectangles; frame k
    is seen by camera k.  The camera advances 0.05 per frame along its view
    axis with a slow sideways drift and a yaw of about 0.01 rad per frame.
    History depth intervals are drawn around depth 4 with widths 0.5 to 3;
    query tokens draw their depth around the block's own interval, a block-wise
    fraction of them (0 to 15 %) are holes.  ``b`` may be less than the
    rectangle's token count (the first b tokens, row-major, are kept).
    """
    rng = np.random.default_rng(seed)
    fh, fw = frame_hw
    bh, bw = block_hw
    assert fh % bh == 0 and fw % bw == 0 and b <= bh * bw
    per_frame = (fh // bh) * (fw // bw)
    n_hf = -(-M // per_frame)
    n_qf = -(-N // per_frame)
    n_cams = n_hf + n_qf

    cams = np.zeros((n_cams, 16), dtype=np.float32)
    f = 0.75 * fw
    for k in range(n_cams):
        R = _yaw(0.01 * k + 0.002 * rng.standard_normal())
        C = np.array([0.02 * np.sin(0.3 * k), 0.01 * rng.standard_normal(), 0.05 * k])
        cams[k] = [f, f, fw / 2.0, fh / 2.0, *R.reshape(-1), *C]

    def rects(n, first_frame):
        out = np.zeros((n, 4), dtype=np.float32)
        cam = np.zeros(n, dtype=np.int32)
        for j in range(n):
            fr, w = divmod(j, per_frame)
            by, bx = divmod(w, fw // bw)
            out[j] = [bx * bw, (bx + 1) * bw, by * bh, (by + 1) * bh]
            cam[j] = first_frame + fr
        return out, cam

    h_rect, h_cam = rects(M, 0)
    zlo = rng.uniform(2.5, 4.5, size=M)
    zhi = zlo + rng.uniform(0.5, 3.0, size=M)
    h_slab = np.concatenate([h_rect, np.stack([zlo, zhi], 1).astype(np.float32)], 1)
    h_valid = (rng.random(M) >= p_invalid).astype(np.int32)

    q_rect, q_cam = rects(N, n_hf)
    qc = rng.uniform(3.0, 5.0, size=N)
    qw = rng.uniform(0.2, 2.0, size=N)
    q_slab = np.concatenate([q_rect, np.stack([qc - qw / 2, qc + qw / 2], 1).astype(np.float32)], 1)
    q_uvz = np.zeros((N, b, 3), dtype=np.float32)
    for i in range(N):
        t = np.arange(b)
        q_uvz[i, :, 0] = q_rect[i, 0] + (t % bw) + 0.5
        q_uvz[i, :, 1] = q_rect[i, 2] + (t // bw) + 0.5
        z = rng.uniform(qc[i] - 0.6 * qw[i], qc[i] + 0.6 * qw[i], size=b)
        z[rng.random(b) < rng.uniform(0.0, 0.15)] = 0.0
        q_uvz[i, :, 2] = z
    return Scene(cams, q_slab.astype(np.float32), q_cam, q_uvz, h_slab.astype(np.float32), h_cam,
                 h_valid)


def pack_slabs(slab: np.ndarray, cam: np.ndarray, valid=None) -> np.ndarray:
    """[n][8] int32 records: fp32 bits of u0, u1, v0, v1, zlo, zhi; cam; valid."""
    n = slab.shape[0]
    out = np.zeros((n, 8), dtype=np.int32)
    out[:, :6] = np.ascontiguousarray(slab[:, :6], dtype=np.float32).view(np.int32)
    out[:, 6] = cam
    out[:, 7] = 1 if valid is None else valid
    return out


def random_pose_scene(seed: int, N: int, M: int, b: int = 64, frame_hw=(32, 48),
                      n_cams: int = 6, max_angle: float = 0.6,
                      p_invalid: float = 0.1) -> Scene:
    """A scene with arbitrary camera poses, for fuzzing the geometry.

    ``n_cams`` cameras with rotations about random axes by up to
    ``max_angle`` radians (Rodrigues' formula), centres in [-1, 1]^3, focal
    lengths 20-60 and principal points near the frame centre; N query and M
    history slabs with random rectangles (1-16 tokens a side) of random
    cameras, depth intervals starting in [1, 8] with widths 0.2-4; each
    query block's b tokens sit in its rectangle with depths around its
    interval (about 10 % holes).  Seeded numpy, no projection arithmetic.
    """
    rng = np.random.default_rng(seed)
    fh, fw = frame_hw
    cams = np.zeros((n_cams, 16), dtype=np.float32)
    for k in range(n_cams):
        axis = rng.standard_normal(3)
        axis /= np.linalg.norm(axis)
        ang = rng.uniform(-max_angle, max_angle)
        Kx = np.array([[0.0, -axis[2], axis[1]], [axis[2], 0.0, -axis[0]],
                       [-axis[1], axis[0], 0.0]])
        R = np.eye(3) + np.sin(ang) * Kx + (1.0 - np.cos(ang)) * Kx @ Kx
        C = rng.uniform(-1.0, 1.0, size=3)
        f = rng.uniform(20.0, 60.0, size=2)
        cx, cy = fw / 2.0 + rng.uniform(-4.0, 4.0), fh / 2.0 + rng.uniform(-3.0, 3.0)
        cams[k] = [f[0], f[1], cx, cy, *R.reshape(-1), *C]

    def slabs(n):
        w = rng.integers(1, min(16, fw) + 1, size=n)
        h = rng.integers(1, min(16, fh) + 1, size=n)
        u0 = rng.integers(0, fw - w + 1)
        v0 = rng.integers(0, fh - h + 1)
        zlo = rng.uniform(1.0, 8.0, size=n)
        zhi = zlo + rng.uniform(0.2, 4.0, size=n)
        sl = np.stack([u0, u0 + w, v0, v0 + h, zlo, zhi], 1).astype(np.float32)
        return sl, rng.integers(0, n_cams, size=n).astype(np.int32)

    h_slab, h_cam = slabs(M)
    h_valid = (rng.random(M) >= p_invalid).astype(np.int32)
    q_slab, q_cam = slabs(N)
    q_uvz = np.zeros((N, b, 3), dtype=np.float32)
    for i in range(N):
        u0, u1, v0, v1, zlo, zhi = (float(x) for x in q_slab[i])
        q_uvz[i, :, 0] = rng.uniform(u0, u1, size=b)
        q_uvz[i, :, 1] = rng.uniform(v0, v1, size=b)
        z = rng.uniform(zlo - 0.3, zhi + 0.3, size=b)
        z[rng.random(b) < 0.1] = 0.0
        q_uvz[i, :, 2] = z
    return Scene(cams, q_slab, q_cam, q_uvz, h_slab, h_cam, h_valid)


def random_depth_maps(seed: int, n_frames: int, H: int, W: int, s: int = 1,
                      p_hole: float = 0.1) -> np.ndarray:
    """[n_frames][H s][W s] fp32 depths drawn uniformly from [2, 8], a
    fraction p_hole of them 0 (no depth): source maps for fuzzing the
    multiwarp with the cameras of random_pose_scene."""
    rng = np.random.default_rng(seed)
    d = rng.uniform(2.0, 8.0, size=(n_frames, H * s, W * s)).astype(np.float32)
    d[rng.random(d.shape) < p_hole] = 0.0
    return d
