"""Pins of the audit oracle (R_geo, R_50, top-80 recall, changed blocks).

The printed random expectation 50/143 = 0.350 (tests/golden) is met by
independent random p and g; the closed forms g = p (R_50 = 1), positive set =
model top-50 (R_geo = 1) and its complement (R_geo = 0), lambda = 0 (fusion
changes nothing), K >= M (everything selected); the invariant that fusion can
only add positive blocks to a top-K (it raises positive blocks and leaves the
others); top-K against numpy's lexsort; the fused top-K against the route
build's pure top-K (theta > 1, nothing reserved).
"""

import os

import numpy as np
import pytest

from oracle import audit as oa
from oracle import route as ort

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "audit_random_expectation.txt")


def _golden():
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            k, M, e = line.split()
            return int(k), int(M), float(e)


def _softmax_rows(x):
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)


def _g_audit(rng, N, M):
    # audit-style overlap: 10 % of the blocks positive, U[0.2, 1]
    g = np.where(rng.random((N, M)) < 0.1, 0.2 + 0.8 * rng.random((N, M)), 0.0)
    return g.astype(np.float32)


def test_random_expectation_matches_printed_value():
    k, M, printed = _golden()
    assert abs(k / M - printed) < 5e-4
    rng = np.random.default_rng(11)
    N = 400
    p = _softmax_rows(rng.standard_normal((1, N, M)))
    g = _g_audit(rng, N, M)
    c = oa.audit(p, g, ort.Params(), k_geo=k, k_fuse=80)
    m = oa.metrics(c, M, k, 80)
    n_pos = c[..., 0].sum()
    sd_geo = np.sqrt(k / M * (1 - k / M) / n_pos)
    sd_50 = np.sqrt(k / M * (1 - k / M) / (N * k))
    assert abs(m.R_geo - k / M) < 4 * sd_geo
    assert abs(m.R_50 - k / M) < 4 * sd_50


def test_closed_forms():
    rng = np.random.default_rng(2)
    M = 143
    p = _softmax_rows(rng.standard_normal((1, 3, M)))
    # g ranks exactly like p -> top-50 agreement 1
    c = oa.audit(p, p[0].copy(), ort.Params(), 50, 80)
    assert np.all(c[..., 2] == 50)
    # positives = the model's own top-50 -> R_geo = 1; the complement -> 0
    g = np.zeros((3, M), np.float32)
    for i in range(3):
        g[i, sorted(oa.top_k(p[0, i], 50))] = 0.5
    c = oa.audit(p, g, ort.Params(), 50, 80)
    assert oa.metrics(c, M).R_geo == 1.0
    c = oa.audit(p, np.where(g > 0, 0.0, 0.5).astype(np.float32), ort.Params(), 50, 80)
    assert oa.metrics(c, M).R_geo == 0.0


def test_lambda_zero_changes_nothing_and_k_ge_m_takes_all():
    rng = np.random.default_rng(3)
    M = 60
    p = _softmax_rows(rng.standard_normal((2, 5, M)))
    g = _g_audit(rng, 5, M)
    c = oa.audit(p, g, ort.Params(lam=0.0), 50, 30)
    assert np.all(c[..., 3] == c[..., 4]) and np.all(c[..., 5] == 0)
    c = oa.audit(p, g, ort.Params(), 60, 200)
    m = oa.metrics(c, M, 60, 200)
    assert m.R_geo == 1.0 and m.R_50 == 1.0 and m.changed == 0.0


def test_fusion_only_adds_positive_blocks():
    rng = np.random.default_rng(4)
    M = 143
    p = _softmax_rows(2.0 * rng.standard_normal((4, 12, M)))
    g = _g_audit(rng, 12, M)
    c = oa.audit(p, g, ort.Params(lam=2.0), 50, 80)
    assert np.all(c[..., 4] >= c[..., 3])
    assert np.any(c[..., 4] > c[..., 3])
    assert np.all(c[..., 5] <= 80)


def test_top_k_against_lexsort_with_ties():
    rng = np.random.default_rng(5)
    for M in (1, 7, 50, 143):
        s = rng.integers(0, 5, size=M).astype(np.float64)   # many ties
        order = np.lexsort((np.arange(M), -s))
        for K in (1, 3, M, M + 4):
            assert oa.top_k(s, K) == set(order[:K].tolist())


def test_fused_top_k_equals_pure_top_k_route():
    rng = np.random.default_rng(6)
    M = 143
    p = _softmax_rows(rng.standard_normal((1, 6, M)))[0]
    g = _g_audit(rng, 6, M)
    prm = ort.Params(theta_cov=2.0, k_cov=80)
    for i in range(6):
        budget, _, _ = ort.route_row(p[i], g[i], True, prm, 0, 0)
        assert set(budget) == oa.top_k(ort.fused_weight(p[i], g[i], prm), 80)


def test_positive_overlap_is_strictly_above_tau():
    # g == tau is not a positive block (strict >, as printed for g^)
    M = 20
    p = _softmax_rows(np.random.default_rng(7).standard_normal((1, 1, M)))
    g = np.zeros((1, M), np.float32)
    g[0, :5] = np.float32(0.1)
    g[0, 5:8] = np.nextafter(np.float32(0.1), np.float32(1))
    c = oa.audit(p, g, ort.Params(tau=0.1), 5, 8)
    assert c[0, 0, 0] == 3


def test_metrics_pool_rows_and_changed_is_against_the_model_top_k():
    # R_geo is a ratio of sums over rows (10 / 12), not a mean of per-row
    # ratios (0.5)
    c = np.zeros((2, 6), dtype=np.int64)
    c[0, :2] = [10, 10]
    c[1, :2] = [2, 0]
    assert oa.metrics(c, 143).R_geo == 10 / 12
    # lambda = 0 with the defaults (top-50 for R_geo, top-80 for the fusion
    # rows): the fused top-80 is the model's top-80, nothing changes
    rng = np.random.default_rng(8)
    M = 143
    p = _softmax_rows(rng.standard_normal((1, 4, M)))
    g = _g_audit(rng, 4, M)
    c = oa.audit(p, g, ort.Params(lam=0.0))
    assert np.all(c[..., 5] == 0) and oa.metrics(c, M).changed == 0.0
