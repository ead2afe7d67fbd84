"""Pins of the oracle's frustum-slab overlap and coverage.

Checked against closed forms that the geometry fixes: identical slabs overlap
fully, far-apart slabs not at all; two equal boxes shifted by k grid cells
along an axis have IoU f / (2 - f) with f = 1 - k/G exactly (the grid
samples sit half a cell away from every face); a slab inside a larger one has
IoU = volume ratio; a rigid motion of the whole scene changes nothing; a
token inside (outside) a slab's rectangle and depth range, seen from the same
or from another camera, is (is not) covered.
"""

import numpy as np
import pytest

from oracle import geometry as geo


def cam(fx=2.0, fy=2.0, cx=4.0, cy=4.0, R=None, C=(0.0, 0.0, 0.0)):
    R = np.eye(3) if R is None else np.asarray(R)
    return np.array([fx, fy, cx, cy, *R.reshape(-1), *C], dtype=np.float32)


def rot(axis, ang):
    a = np.asarray(axis, dtype=np.float64)
    a = a / np.linalg.norm(a)
    K = np.array([[0, -a[2], a[1]], [a[2], 0, -a[0]], [-a[1], a[0], 0]])
    return np.eye(3) + np.sin(ang) * K + (1 - np.cos(ang)) * K @ K


SLAB = np.array([2.0, 6.0, 2.0, 6.0, 3.0, 5.0], dtype=np.float32)  # zm = 4, half 4x4x1


def test_obb_closed_form():
    c, R, h = geo.obb(cam(), SLAB)
    # centre ray through (4, 4) = principal point, mid depth 4
    assert np.allclose(c, [0, 0, 4]) and np.allclose(h, [4, 4, 1]) and np.allclose(R, np.eye(3))


def test_identical_and_disjoint_slabs():
    assert geo.slab_iou(cam(), SLAB, cam(), SLAB, True, 6) == 1.0
    far = cam(C=(100.0, 0.0, 0.0))
    assert geo.slab_iou(cam(), SLAB, far, SLAB, True, 6) == 0.0
    assert geo.slab_iou(cam(), SLAB, cam(), SLAB, False, 6) == 0.0


@pytest.mark.parametrize("G,k", [(4, 1), (8, 3), (8, 7), (6, 2)])
def test_shifted_equal_boxes_exact_iou(G, k):
    # box half extent along x is 4: a shift of k cells is 8 k / G
    shift = 8.0 * k / G
    g = geo.slab_iou(cam(), SLAB, cam(C=(shift, 0.0, 0.0)), SLAB, True, G)
    f = 1.0 - k / G
    assert abs(g - f / (2.0 - f)) < 1e-12


def test_nested_box_is_volume_ratio():
    big = np.array([0.0, 8.0, 0.0, 8.0, 2.0, 6.0], dtype=np.float32)  # zm 4: half 8x8x2
    g = geo.slab_iou(cam(), SLAB, cam(), big, True, 8)
    assert abs(g - (4 * 4 * 1) / (8 * 8 * 2)) < 1e-12


def test_rigid_motion_of_the_scene_changes_nothing():
    Rg = rot([1.0, 2.0, 0.5], 0.7)
    t = np.array([3.0, -1.0, 2.0])
    c0 = cam(R=Rg, C=tuple(t))
    c1 = cam(R=Rg, C=tuple(t + Rg @ np.array([8.0 * 3 / 8, 0.0, 0.0])))
    g = geo.slab_iou(c0, SLAB, c1, SLAB, True, 8)
    f = 1.0 - 3 / 8
    assert abs(g - f / (2.0 - f)) < 1e-6


def test_token_inside_same_camera():
    c = cam()
    inside = [(2.5, 2.5, 3.5), (5.9, 5.0, 5.0), (2.0, 2.0, 3.0)]
    outside = [(6.0, 3.0, 4.0), (3.0, 3.0, 5.5), (3.0, 3.0, 2.9), (3.0, 3.0, 0.0), (3.0, 3.0, -4.0)]
    for u, v, z in inside:
        assert geo.token_inside(c, u, v, z, c, SLAB)
    for u, v, z in outside:
        assert not geo.token_inside(c, u, v, z, c, SLAB)


def test_token_seen_from_another_camera():
    # camera 1 sits 2 units to the right of camera 0 with the same orientation:
    # a world point at (x, y, z) is pixel u1 = (x - 2) / z * fx + cx in it
    c0, c1 = cam(), cam(C=(2.0, 0.0, 0.0))
    # token of camera 1 at u = 3, v = 4, depth 4 -> world x = (3 - 4) / 2 * 4 + 2 = 0
    # -> pixel (4, 4) in camera 0, depth 4: inside SLAB
    assert geo.token_inside(c1, 3.0, 4.0, 4.0, c0, SLAB)
    # the same token at depth 8 leaves SLAB's depth range
    assert not geo.token_inside(c1, 3.0, 4.0, 8.0, c0, SLAB)


def test_coverage_fraction_and_threshold():
    cams = [cam()]
    b = 10
    uvz = np.zeros((2, b, 3), dtype=np.float32)
    uvz[:, :, 0] = 3.0
    uvz[:, :, 1] = 3.0
    uvz[0, :, 2] = 4.0           # all 10 tokens inside
    uvz[1, :, 2] = 4.0
    uvz[1, :2, 2] = 9.0          # 8 of 10 inside
    rho, cov = geo.coverage(cams, [0, 0], uvz, [0], [SLAB], [1], eta=0.9)
    assert rho.tolist() == [1.0, 0.8] and cov.tolist() == [1, 0]
    rho, cov = geo.coverage(cams, [0, 0], uvz, [0], [SLAB], [0], eta=0.9)
    assert rho.tolist() == [0.0, 0.0]


# ---- marginal decisions: the count interval [n_lo, n_hi] ----

def test_grid_points_on_a_face_are_marginal():
    # G = 4: the query box's samples sit at x in {-3, -1, 1, 3}.  The history
    # box (half extent 4) shifted by 1 has its face at x = -3: one plane of
    # 16 samples lies exactly on it (inside by definition, |d| <= h), so the
    # fp64 count is 64, but another precision may put those 16 either side.
    n, lo, hi, vi, vr = geo.slab_iou_counts(cam(), SLAB, cam(C=(1.0, 0.0, 0.0)), SLAB, True, 4)
    assert (n, lo, hi) == (64, 48, 64)
    # moved a thousandth further the plane is clearly outside: no margin case
    n, lo, hi, _, _ = geo.slab_iou_counts(cam(), SLAB, cam(C=(1.001, 0.0, 0.0)), SLAB, True, 4)
    assert (n, lo, hi) == (48, 48, 48)
    g, g_lo, g_hi = geo.overlap_bounds([cam(), cam(C=(1.0, 0.0, 0.0))], [0], [SLAB], [1],
                                       [SLAB], [1], 4)
    assert g_lo[0, 0] < g[0, 0] == g_hi[0, 0] == 1.0


@pytest.mark.parametrize("G,k", [(4, 1), (8, 3)])
def test_whole_cell_shifts_have_no_marginal_samples(G, k):
    # samples sit half a cell from every face: the count is fixed
    n, lo, hi, _, _ = geo.slab_iou_counts(cam(), SLAB, cam(C=(8.0 * k / G, 0.0, 0.0)), SLAB,
                                          True, G)
    assert n == lo == hi == G * G * (G - k)


def test_token_on_a_rectangle_edge_is_marginal():
    c = cam()
    X = geo.token_world(c, 2.0, 3.0, 4.0)        # u exactly on the edge u0 = 2
    inside, margin = geo.inside_margin(X, c, SLAB)
    assert inside and margin == 0.0
    uvz = np.array([[[2.0, 3.0, 4.0], [3.0, 3.0, 4.0], [1.5, 3.0, 4.0], [1.99, 3.0, 4.0]]],
                   dtype=np.float32)
    n, lo, hi = geo.coverage_bounds([c], [0], uvz, [0], [SLAB], [1])
    # edge token: counted, marginal; (3, 3): inside by 1 token = 2 world
    # units at depth 4; (1.5, 3) and (1.99, 3): outside by 0.5 and 0.01
    # tokens (1 and 0.02 world units): both clear of the margin
    assert (n[0], lo[0], hi[0]) == (2, 1, 2)


def test_coverage_count_faces_half_open_rectangle_closed_depth():
    # The coverage count of a token on each face of SLAB, with exactly
    # representable coordinates (fx = 2, cx = 4, R = I: token (u, v, z)
    # projects back to (u, v) at depth z with no rounding): the rectangle is
    # [u0, u1) x [v0, v1), the depth interval [z-, z+].
    c = cam()
    faces = [((2.0, 3.0, 4.0), True),    # u = u0
             ((6.0, 3.0, 4.0), False),   # u = u1
             ((3.0, 2.0, 4.0), True),    # v = v0
             ((3.0, 6.0, 4.0), False),   # v = v1
             ((3.0, 3.0, 3.0), True),    # z = z-
             ((3.0, 3.0, 5.0), True)]    # z = z+
    uvz = np.array([[t for t, _ in faces]], dtype=np.float32).reshape(len(faces), 1, 3)
    n, _, _ = geo.coverage_bounds([c], [0] * len(faces), uvz, [0], [SLAB], [1])
    assert n.tolist() == [int(want) for _, want in faces]
    for (u, v, z), want in faces:
        assert geo.token_inside(c, u, v, z, c, SLAB) == want


def test_covered_when_rho_equals_eta():
    # rho = 2 / 4 = eta = 0.5 exactly: covered (rho >= eta)
    uvz = np.zeros((1, 4, 3), dtype=np.float32)
    uvz[0, :, :2] = 3.0
    uvz[0, :, 2] = [4.0, 4.0, 9.0, 9.0]
    rho, cov = geo.coverage([cam()], [0], uvz, [0], [SLAB], [1], eta=0.5)
    assert rho.tolist() == [0.5] and cov.tolist() == [1]


def test_coverage_upper_count_holds_tokens_just_outside():
    # a token exactly on the far face u = u1 is outside (the rectangle is
    # half-open) but within the marginal distance: n_hi counts it, n does not
    c = cam()
    uvz = np.array([[[6.0, 3.0, 4.0]], [[3.0, 6.0, 4.0]], [[7.0, 3.0, 4.0]]], dtype=np.float32)
    n, lo, hi = geo.coverage_bounds([c], [0, 0, 0], uvz, [0], [SLAB], [1])
    assert n.tolist() == [0, 0, 0] and lo.tolist() == [0, 0, 0] and hi.tolist() == [1, 1, 0]
