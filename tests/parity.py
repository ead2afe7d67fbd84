"""Comparison helpers shared by the GPU parity tests.

Tolerances (written out here, derived in the design notes):

* Gilbert ranks, block ids, neighbour ids, route ids: bit-exact.  A route may
  differ from the oracle's only at its mass cut and only when the oracle's
  cumulative mass there lies within MASS_EPS of theta (fp64 sums in a
  different order), by one block at the cut.
* block importance p: fp32 pooling / dot products / exp against fp64, so
  |p_gpu / p_ref - 1| <= P_RTOL.
* slab overlap g: the inside counts must agree exactly; the fp32 volume and
  ratio arithmetic adds a few ulps, and a count off by one moves g by at least
  1/G^3 >= 3e-5 relative (G <= 32), so |g_gpu / g_ref - 1| <= G_RTOL = 4e-6
  separates the two.  Coverage rho and the covered flags: exact.
* attention O: bf16 inputs, fp32 accumulation, bf16 P and bf16 output:
  max |O_gpu - O_ref| <= 2e-2 and sum |O_gpu - O_ref| / sum |O_ref| <= 5e-3;
  lse within LSE_ATOL.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oatt
from oracle import importance as oimp
from oracle import route as ort

MASS_EPS = 1e-11
P_RTOL = 2e-5
O_MAX_ABS = 2e-2
O_MEAN_REL = 5e-3
LSE_ATOL = 1e-3
G_RTOL = 4e-6


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_params(prm) -> ort.Params:
    return ort.Params(lam=prm.lam, tau=prm.tau, g_ref=prm.g_ref, theta_cov=prm.theta_cov,
                      theta_unc=prm.theta_unc, k_cov=prm.k_cov, k_unc=prm.k_unc)


def oracle_importance(Q, K, heads, scale=1.0, b=128):
    return {h: oimp.importance(f64(Q[h]), f64(K[h]), b, scale) for h in heads}


def oracle_routes(p_rows, g, covered, prm, prev_begin, prev_count, nbr=None, ref=()):
    """p_rows: {h: [N][M] array (fp32 values)} -> {(h, i): (budget, extras, info)}."""
    out = {}
    N = g.shape[0]
    for h, ph in p_rows.items():
        for i in range(N):
            safe = list(nbr[i]) if nbr is not None else []
            safe += list(ref)
            out[(h, i)] = ort.route_row(ph[i], g[i], bool(covered[i]), prm, prev_begin,
                                        prev_count, safe)
    return out


def gpu_row(route_ids, route_len, route_nb, h, i):
    L = int(route_len[h, i])
    nb = int(route_nb[h, i])
    ids = route_ids[h, i].tolist()
    return ids[:nb], ids[nb:L], ids[L:]


def check_route_row(gpu, ref, where=""):
    """Returns 'exact' or 'cut' (an allowed one-block difference at the cut)."""
    g_budget, g_extra, g_pad = gpu
    budget, extras, info = ref
    assert all(x == -1 for x in g_pad), f"{where}: padding {g_pad[:8]}"
    assert g_budget == sorted(g_budget) and g_extra == sorted(g_extra), where
    if g_budget == budget:
        assert g_extra == extras, f"{where}: extras {g_extra} != {extras}"
        return "exact"
    near = abs(info["mass_at_cut"] - info["theta"]) <= MASS_EPS
    assert near, f"{where}: budget differs ({len(g_budget)} vs {len(budget)}) away from the cut"
    a, b = set(g_budget), set(budget)
    assert len(a ^ b) == 1, f"{where}: more than one block differs at the cut"
    return "cut"


def attention_rows(Q, K, V, rows, tiles_of, scale=0.0, b=128):
    """Oracle O and lse for the (h, i) rows; tiles_of(h, i) -> tile ids."""
    out = {}
    cache = {}
    for (h, i) in rows:
        if h not in cache:
            cache.clear()
            cache[h] = (f64(K[h]), f64(V[h]))
        Kh, Vh = cache[h]
        q = f64(Q[h, i * b:(i + 1) * b])
        out[(h, i)] = oatt.routed_attention_block(q, Kh, Vh, tiles_of(h, i), b, scale)
    return out


def attention_errors(O_gpu, lse_gpu, ref, b=128):
    num = den = 0.0
    worst = 0.0
    worst_lse = 0.0
    for (h, i), (O, lse) in ref.items():
        g = f64(O_gpu[h, i * b:(i + 1) * b])
        diff = np.abs(g - O)
        worst = max(worst, float(diff.max()))
        num += float(diff.sum())
        den += float(np.abs(O).sum())
        if lse_gpu is not None:
            gl = f64(lse_gpu[h, i * b:(i + 1) * b])
            fin = np.isfinite(lse)
            assert np.array_equal(np.isfinite(gl), fin)
            if fin.any():
                worst_lse = max(worst_lse, float(np.abs(gl[fin] - lse[fin]).max()))
    mean_rel = num / den if den > 0 else num
    return worst, mean_rel, worst_lse


def assert_attention_close(O_gpu, lse_gpu, ref, b=128):
    worst, mean_rel, worst_lse = attention_errors(O_gpu, lse_gpu, ref, b)
    assert worst <= O_MAX_ABS, f"max abs err {worst}"
    assert mean_rel <= O_MEAN_REL, f"mean rel err {mean_rel}"
    assert worst_lse <= LSE_ATOL, f"lse err {worst_lse}"
    return worst, mean_rel, worst_lse
