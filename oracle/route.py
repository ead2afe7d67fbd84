"""Soft geometry fusion and route materialisation (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Passages followed:

* fusion: p~_{i,r} is proportional to p_{i,r} (1 + lambda g^_{i,r}) with
  g^ = [g > tau] min(g / g_ref, 1) (Velox project page, "02 · Method", the
  fusion formula and its glossary), applied to covered query blocks only;
  uncovered blocks keep the unbiased p (project page, "Covered and uncovered
  blocks"; onedev.kr summary, "How it differs"; digest of arXiv 2610.22311,
  "Core method", Eq. 11);
* route: renormalise, sort descending, take the minimal prefix whose
  cumulative mass reaches the threshold, capped at K_cov (covered) or K_unc
  (uncovered); previous-chunk blocks are reserved inside the budget; the
  Gilbert 26-neighbour blocks and reference blocks are appended outside it
  (digest, "Method steps", step four, Eq. 12-14; onedev.kr summary, "How it
  differs").

Readings where the pages are open:

* the mass threshold is theta_cov for covered and theta_unc for uncovered
  rows; "reaches" means cumulative mass >= theta;
* reserved blocks come first in the walk: they always enter the budget, their
  count counts toward K and their mass toward theta; if they alone fill K or
  reach theta nothing else is added;
* ties in the descending sort go to the lower block id;
* the sort key is the unnormalised fused weight w_r = p_r (1 + lambda g^_r)
  (p_r on uncovered rows).  Dividing by the positive row sum does not change
  the order, and keying on w keeps the order independent of how the row sum
  is rounded;
* every floating-point step is fp64 from the fp32 inputs, with the fp32
  parameters lambda, tau, g_ref, theta converted exactly; g > tau is a strict
  comparison, as printed;
* output: the budget ids ascending, then the safeguard/reference ids not
  already in the budget, ascending and without repeats.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Iterable, List, Sequence, Tuple

import numpy as np


@dataclass(frozen=True)
class Params:
    lam: float = 2.0
    tau: float = 0.1
    g_ref: float = 0.2
    theta_cov: float = 0.9
    theta_unc: float = 0.9
    k_cov: int = 80
    k_unc: int = 150


def _f32(v: float) -> float:
    """The fp64 value of v rounded to fp32, as the parameters travel in fp32."""
    return float(np.float32(v))


def fused_weight(p_row: np.ndarray, g_row: np.ndarray, prm: Params) -> np.ndarray:
    """w_r = p_r * (1 + lambda * g^_r), g^_r = [g_r > tau] * min(g_r / g_ref, 1)."""
    p = np.asarray(p_row, dtype=np.float32).astype(np.float64)
    g = np.asarray(g_row, dtype=np.float32).astype(np.float64)
    ghat = np.where(g > _f32(prm.tau), np.minimum(g / _f32(prm.g_ref), 1.0), 0.0)
    return p * (1.0 + _f32(prm.lam) * ghat)


def route_row(p_row, g_row, covered: bool, prm: Params, prev_begin: int,
              prev_count: int, safeguards: Iterable[int] = ()) -> Tuple[List[int], List[int], dict]:
    """Route of one (head, query block) row.

    Returns (budget ids ascending, extra ids ascending, info) where info holds
    the fp64 scores s, the walk order, and the cumulative mass at the cut.
    """
    p = np.asarray(p_row, dtype=np.float32).astype(np.float64)
    M = p.shape[0]
    if covered:
        key = fused_weight(p_row, g_row, prm)
        s = key / key.sum()
        K, theta = prm.k_cov, _f32(prm.theta_cov)
    else:
        key = p
        s = p
        K, theta = prm.k_unc, _f32(prm.theta_unc)
    reserved = list(range(prev_begin, prev_begin + prev_count))
    is_res = np.zeros(M, dtype=bool)
    is_res[reserved] = True
    ids = np.arange(M)
    rest = ids[~is_res]
    # descending key, ties by ascending id (lexsort: last key is primary)
    rest = rest[np.lexsort((rest, -key[rest]))]
    budget = list(reserved)
    mass = 0.0
    for r in reserved:
        mass += s[r]
    walked = 0
    for r in rest:
        if len(budget) >= K or mass >= theta:
            break
        budget.append(int(r))
        mass += s[r]
        walked += 1
    bset = set(budget)
    extras = sorted(set(int(u) for u in safeguards) - bset)
    info = {"s": s, "key": key, "order": rest, "n_walked": walked,
            "mass_at_cut": mass, "theta": theta, "K": K}
    return sorted(budget), extras, info


def route_build(p: np.ndarray, g: np.ndarray, covered: Sequence[int], prm: Params,
                prev_begin: int, prev_count: int,
                nbr: Sequence[Sequence[int]] = (), ref: Sequence[int] = ()):
    """Routes of every row of one head: p [N][M], g [N][M], covered [N].

    nbr[i] are the 26-neighbour cache ids of query block i (may be empty).
    Returns a list of (budget, extras, info) per row.
    """
    N = p.shape[0]
    out = []
    for i in range(N):
        safe = list(nbr[i]) if len(nbr) else []
        safe += list(ref)
        out.append(route_row(p[i], g[i], bool(covered[i]), prm, prev_begin,
                             prev_count, safe))
    return out
