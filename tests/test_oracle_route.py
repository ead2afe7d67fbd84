"""Pins of the oracle's soft fusion and route materialisation.

Checked against what the pages fix (Velox project page, "02 · Method": fusion
formula, "a vetted block gains at most 3x", "Covered and uncovered blocks";
arXiv 2610.22311 digest, "Method steps", Eq. 12-14; onedev.kr summary, "How
it differs") and against brute force:

* the hand-derived multiplier table in tests/golden/fusion_multiplier.txt;
* lambda = 0, g = 0, or an uncovered row reproduce the model-only route;
* a threshold above 1 gives the exact top-K (heapq, a different routine);
* a minimal-cardinality / maximal-mass subset search on rows of <= 10 blocks;
* reserved blocks always enter, count toward K and toward the mass;
* safeguards are appended outside the budget, once, ascending.
"""

import heapq
import itertools
import os

import numpy as np
import pytest

from oracle import route as rt

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fusion_multiplier.txt")


def _row(seed, M, peaked=1.0):
    r = np.random.default_rng(seed)
    x = r.standard_normal(M) * peaked
    p = np.exp(x - x.max())
    p = (p / p.sum()).astype(np.float32)
    g = r.random(M).astype(np.float32)
    g[r.random(M) < 0.5] = 0.0
    return p, g


def test_fusion_multiplier_golden_table():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    prm = rt.Params()
    g = np.array([float(r[0]) for r in rows], dtype=np.float32)
    want = np.array([float(r[2]) for r in rows])
    w = rt.fused_weight(np.ones_like(g), g, prm)
    assert np.allclose(w, want, rtol=0, atol=1e-6)
    assert w.max() == 3.0 and w.min() == 1.0


def test_multiplier_bounded_by_one_plus_lambda():
    for seed in range(5):
        p, g = _row(seed, 300)
        for lam in (0.5, 2.0, 7.0):
            prm = rt.Params(lam=lam)
            ratio = rt.fused_weight(p, g, prm) / p.astype(np.float64)
            assert ratio.min() >= 1.0 and ratio.max() <= 1.0 + np.float32(lam)


@pytest.mark.parametrize("variant", ["lambda0", "g0"])
def test_no_geometry_reproduces_model_only_route(variant):
    for seed in range(8):
        p, g = _row(seed, 200, peaked=3.0)
        prm = rt.Params(k_cov=60, k_unc=60, theta_cov=0.8, theta_unc=0.8,
                        lam=0.0 if variant == "lambda0" else 2.0)
        if variant == "g0":
            g = np.zeros_like(g)
        cov = rt.route_row(p, g, True, prm, 190, 10)
        unc = rt.route_row(p, g, False, prm, 190, 10)
        # the covered row renormalises p, which can move the cut by rounding
        # only when the mass lands within an ulp of theta
        if abs(unc[2]["mass_at_cut"] - unc[2]["theta"]) > 1e-12:
            assert cov[0] == unc[0]


def test_threshold_above_one_is_exact_top_k():
    for seed in range(10):
        M = 120
        p, g = _row(seed, M)
        p[5] = p[9]          # an exact tie: the lower id must win
        prm = rt.Params(theta_cov=2.0, theta_unc=2.0, k_cov=30, k_unc=45)
        for covered in (True, False):
            budget, _, info = rt.route_row(p, g, covered, prm, 100, 20)
            K = 30 if covered else 45
            key = info["key"]
            rest = [r for r in range(M) if not 100 <= r < 120]
            top = heapq.nlargest(K - 20, rest, key=lambda r: (key[r], -r))
            assert budget == sorted(list(range(100, 120)) + top)


def test_cap_at_least_M_takes_everything():
    p, g = _row(3, 50)
    prm = rt.Params(theta_cov=1.5, theta_unc=1.5, k_cov=50, k_unc=80)
    for covered in (True, False):
        budget, _, _ = rt.route_row(p, g, covered, prm, 45, 5)
        assert budget == list(range(50))


def test_reserved_rules():
    p, g = _row(4, 40)
    # |P| >= K: the budget is exactly P
    prm = rt.Params(k_cov=3, k_unc=3)
    assert rt.route_row(p, g, False, prm, 30, 6)[0] == list(range(30, 36))
    # mass(P) >= theta: nothing else is added
    q = np.full(40, 1e-4, dtype=np.float32)
    q[10:14] = (1.0 - 36e-4) / 4
    assert rt.route_row(q, g, False, rt.Params(), 10, 4)[0] == [10, 11, 12, 13]
    # P always present, counted in K
    budget, _, _ = rt.route_row(p, g, True, rt.Params(k_cov=10, theta_cov=2.0), 0, 4)
    assert budget[:4] == [0, 1, 2, 3] and len(budget) == 10


def _brute(s, key, P, K, theta, M):
    """Smallest budget S >= P (|S| <= max(K, |P|)) with mass >= theta, ties to
    the larger mass, then to the lexicographically larger keys/smaller ids."""
    others = [r for r in range(M) if r not in P]
    base = sum(s[r] for r in P)
    if len(P) >= K or base >= theta:
        return sorted(P)
    for m in range(0, K - len(P) + 1):
        best = None
        for extra in itertools.combinations(others, m):
            mass = base + sum(s[r] for r in extra)
            if mass >= theta or m == K - len(P):
                cand = (sorted(((key[r], -r) for r in extra), reverse=True), extra)
                if best is None or cand[0] > best[0]:
                    best = cand
        if best is not None:
            return sorted(list(P) + list(best[1]))
    raise AssertionError


@pytest.mark.parametrize("M", [4, 6, 8, 10])
def test_brute_force_minimal_prefix(M):
    r = np.random.default_rng(M)
    for trial in range(40):
        x = r.standard_normal(M) * r.uniform(0.2, 4.0)
        p = np.exp(x - x.max())
        p = (p / p.sum()).astype(np.float32)
        g = (r.random(M) * (r.random(M) < 0.6)).astype(np.float32)
        nres = int(r.integers(0, 3))
        P = list(range(M - nres, M))
        theta = float(r.uniform(0.3, 0.99))
        K = int(r.integers(max(1, nres), M + 1))
        prm = rt.Params(k_cov=K, k_unc=K, theta_cov=theta, theta_unc=theta)
        for covered in (True, False):
            budget, _, info = rt.route_row(p, g, covered, prm, M - nres, nres)
            if abs(info["mass_at_cut"] - info["theta"]) < 1e-12:
                continue
            assert budget == _brute(info["s"], info["key"], P, K, info["theta"], M)


def test_relabelling_blocks_relabels_the_route():
    M = 64
    p, g = _row(11, M, peaked=2.0)
    sigma = np.random.default_rng(1).permutation(M - 8)   # keep P = last 8 fixed
    sigma = np.concatenate([sigma, np.arange(M - 8, M)])
    inv = np.argsort(sigma)
    prm = rt.Params(k_cov=20, k_unc=30, theta_cov=0.6, theta_unc=0.6)
    for covered in (True, False):
        a = rt.route_row(p, g, covered, prm, M - 8, 8)[0]
        b = rt.route_row(p[sigma], g[sigma], covered, prm, M - 8, 8)[0]
        assert sorted(int(sigma[x]) for x in b) == a
        assert sorted(int(inv[x]) for x in a) == b


def test_safeguards_outside_budget_deduplicated():
    p, g = _row(12, 30)
    prm = rt.Params(k_cov=5, k_unc=5, theta_cov=2.0, theta_unc=2.0)
    budget, extras, _ = rt.route_row(p, g, False, prm, 28, 2, [0, 29, 3, 3, 0, 28, 17])
    assert len(budget) == 5 and 28 in budget and 29 in budget
    want = sorted({0, 3, 17} - set(budget))
    assert extras == want


def test_uncovered_rows_ignore_geometry():
    p, _ = _row(13, 90)
    r = np.random.default_rng(0)
    a = rt.route_row(p, r.random(90).astype(np.float32), False, rt.Params(), 80, 10)[0]
    b = rt.route_row(p, np.zeros(90, np.float32), False, rt.Params(), 80, 10)[0]
    assert a == b


def test_geometry_moves_covered_rows_toward_overlap():
    # A block with full overlap gains exactly 3x before renormalisation; with
    # a flat p and K = |P| + 1 the single extra pick is the overlapping one.
    M = 20
    p = np.full(M, 1.0 / M, dtype=np.float32)
    g = np.zeros(M, dtype=np.float32)
    g[7] = 0.9
    prm = rt.Params(k_cov=3, theta_cov=2.0)
    budget, _, info = rt.route_row(p, g, True, prm, 18, 2)
    assert budget == [7, 18, 19]
    assert abs(info["s"][7] / info["s"][0] - 3.0) < 1e-12


def test_ties_at_the_cut_go_to_lower_ids():
    # A flat row: every non-reserved block ties, so the picks are the lowest ids.
    M = 40
    p = np.full(M, 1.0 / M, dtype=np.float32)
    g = np.zeros(M, dtype=np.float32)
    prm = rt.Params(k_cov=9, k_unc=9, theta_cov=2.0, theta_unc=2.0)
    for covered in (True, False):
        budget, _, _ = rt.route_row(p, g, covered, prm, 35, 5)
        assert budget == [0, 1, 2, 3, 35, 36, 37, 38, 39]
    # ties inside the fused score: g = g_ref and g = 1 give the same multiplier
    g[[30, 12, 20]] = [0.2, 1.0, 0.5]
    budget, _, _ = rt.route_row(p, g, True, rt.Params(k_cov=7, theta_cov=2.0), 35, 5)
    assert budget == [12, 20, 35, 36, 37, 38, 39]


def test_cut_when_mass_reaches_theta_exactly():
    # dyadic masses and theta, all exact in fp32 and fp64: the prefix stops at
    # the first block whose cumulative mass reaches theta (>=), not after it
    p = np.array([0.0625, 0.5, 0.125, 0.25, 0.0625], dtype=np.float32)
    g = np.zeros(5, dtype=np.float32)
    prm = rt.Params(theta_unc=0.75, k_unc=5)
    budget, extras, info = rt.route_row(p, g, False, prm, 0, 0)
    assert budget == [1, 3] and extras == [] and info["mass_at_cut"] == 0.75
    prm = rt.Params(theta_unc=0.875, k_unc=5)
    assert rt.route_row(p, g, False, prm, 0, 0)[0] == [1, 2, 3]
