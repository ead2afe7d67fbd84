"""The random-pose fuzz scenes (synth.geometry.random_pose_scene) exercise
the geometry: seeded, and overlapping and covering somewhere but not
everywhere (checked with the oracle)."""

import numpy as np

from oracle import geometry as geo
from synth.geometry import random_pose_scene


def test_random_pose_scenes_are_seeded_and_not_trivial():
    a, b = random_pose_scene(3, 7, 60, b=64), random_pose_scene(3, 7, 60, b=64)
    assert np.array_equal(a.cams, b.cams) and np.array_equal(a.q_uvz, b.q_uvz)
    pos = cov = tot = 0
    for seed in range(8):
        s = random_pose_scene(seed, 7, 60, b=64)
        ref, _, _ = geo.overlap_bounds(s.cams, s.q_cam, s.q_slab, s.h_cam, s.h_slab, s.h_valid, 4)
        pos += int((ref > 0).sum())
        tot += ref.size
        n, _, _ = geo.coverage_bounds(s.cams, s.q_cam, s.q_uvz, s.h_cam, s.h_slab, s.h_valid)
        cov += int(n.sum())
    assert 0 < pos < tot and 0 < cov < 8 * 7 * 64
