"""Geometry-model consistency audit: recall counts R_geo, R_50, top-K recall.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages state (Velox project page, "03 · Results", "Geometry and the
model agree"; digest of arXiv 2610.22311, "Experiments" and its results
table, row "geometry-model importance consistency audit"; onedev.kr summary,
"Results"):

* R_geo: the blocks with positive slab overlap (g > tau, tau = 0.1) land in
  the model's own top-50 far more often than chance; 0.7302 at layer 14
  against the random expectation 50/143 = 0.350;
* R_50, the top-50 agreement, is 0.8909 at layer 14 against the same random
  expectation 50/143;
* fusion at lambda = 2 raises the top-80 recall of the positive-overlap
  blocks (0.602 -> 0.852) while changing 9.0 % of the selected blocks.

Readings taken where the pages are open:

* "top-K" of a score is its K largest entries, ties to the lower block id
  (as in the route build); K >= M takes every block;
* R_geo = |pos & top50(p)| / |pos| with pos = {r : g_r > tau};
* R_50 = |top50(g) & top50(p)| / 50: the agreement of the geometry's own
  ranking with the model's, the reading under which its random expectation is
  50/143 like R_geo's;
* top-80 recall of a score = |pos & top80(score)| / |pos| for the model's p
  and for the fused weight p (1 + lambda g^) (every row fused: the audit
  measures the fusion rule itself); "changed" = |top80(fused) - top80(p)| / 80;
* a metric over many rows is a ratio of sums over the rows (pooled), so rows
  with no positive block add nothing to R_geo's denominator.

Per row the oracle returns six integers; the metrics are ratios of their sums.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .route import Params, fused_weight

COUNT_NAMES = ("n_pos", "pos_in_top_geo_p", "top_geo_g_in_top_geo_p", "pos_in_top_fuse_p",
               "pos_in_top_fuse_fused", "top_fuse_fused_not_p")


def top_k(score: np.ndarray, K: int) -> set:
    """Ids of the K largest scores, ties to the lower id."""
    M = len(score)
    order = sorted(range(M), key=lambda r: (-float(score[r]), r))
    return set(order[:min(K, M)])


def audit_row(p_row, g_row, prm: Params, k_geo: int = 50, k_fuse: int = 80) -> np.ndarray:
    p = np.asarray(p_row, dtype=np.float32).astype(np.float64)
    g = np.asarray(g_row, dtype=np.float32).astype(np.float64)
    pos = {r for r in range(len(p)) if g[r] > float(np.float32(prm.tau))}
    a_geo, g_geo = top_k(p, k_geo), top_k(g, k_geo)
    a_fuse, f_fuse = top_k(p, k_fuse), top_k(fused_weight(p_row, g_row, prm), k_fuse)
    return np.array([len(pos), len(pos & a_geo), len(g_geo & a_geo), len(pos & a_fuse),
                     len(pos & f_fuse), len(f_fuse - a_fuse)], dtype=np.int64)


def audit(p: np.ndarray, g: np.ndarray, prm: Params, k_geo: int = 50,
          k_fuse: int = 80) -> np.ndarray:
    """counts [H][N][6] for p [H][N][M] and g [N][M]."""
    H, N, _ = p.shape
    out = np.zeros((H, N, 6), dtype=np.int64)
    for h in range(H):
        for i in range(N):
            out[h, i] = audit_row(p[h, i], g[i], prm, k_geo, k_fuse)
    return out


@dataclass
class AuditMetrics:
    R_geo: float
    R_50: float
    recall_fuse_model: float
    recall_fuse_fused: float
    changed: float


def metrics(counts: np.ndarray, M: int, k_geo: int = 50, k_fuse: int = 80) -> AuditMetrics:
    """Pooled ratios over all rows of a counts array [..., 6]."""
    c = np.asarray(counts).reshape(-1, 6).sum(axis=0).astype(np.float64)
    rows = np.asarray(counts).reshape(-1, 6).shape[0]
    n_pos = c[0]
    return AuditMetrics(
        R_geo=c[1] / n_pos if n_pos else float("nan"),
        R_50=c[2] / (rows * min(k_geo, M)),
        recall_fuse_model=c[3] / n_pos if n_pos else float("nan"),
        recall_fuse_fused=c[4] / n_pos if n_pos else float("nan"),
        changed=c[5] / (rows * min(k_fuse, M)),
    )
