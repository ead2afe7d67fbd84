"""Comparison helpers shared by the GPU parity tests.

Tolerances (written out here, derived in the design notes):

* Gilbert ranks, block ids, neighbour ids, route ids: bit-exact.  A route may
  differ from the oracle's only at its mass cut and only when the oracle's
  cumulative mass there lies within MASS_EPS of theta (fp64 sums in a
  different order), by one block at the cut.
* block importance p: fp32 pooling / dot products / exp against fp64, so
  |p_gpu / p_ref - 1| <= P_RTOL.
* slab overlap g, coverage and multiwarp: the oracle decides every
  inside/outside and landing test in fp64 and reports the decisions that
  lie within its marginal distance (oracle.geometry.EPS_REL, 1e-5 of the
  coordinates' size) of a face.  Where no decision of a pair is marginal the
  inside count must agree exactly; the fp32 volume and ratio arithmetic adds
  a few ulps, and a count off by one moves g by at least 1/G^3 >= 3e-5
  relative (G <= 32), so |g_gpu / g_ref - 1| <= G_RTOL = 4e-6 separates the
  two.  Where some are marginal, g_gpu must lie in [g_lo, g_hi] (the values
  of the smallest and largest count the marginal decisions allow), with the
  same slack.  Coverage counts likewise: equal where fixed, within
  [n_lo, n_hi] otherwise.  Multiwarp depths: tokens that no marginal sample
  touches have the same hole pattern and depths within MW_RTOL (the GPU's
  fp32 projection against fp64: a few ulps of coordinates of size ~10 after
  a 3x cancellation, ~2e-6 relative).  Every test counts its marginal cases
  and bounds them by MARGINAL_FRAC of the pairs or tokens (at least 2): the
  bound keeps the oracle from passing a test by calling everything
  marginal; the values themselves are held to the ranges above.
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
MW_RTOL = 1e-5
MARGINAL_FRAC = 0.05
# a marginal sample marks up to 4 candidate tokens, and a small frame takes
# s^2 samples per token from every source: a looser guard for multiwarp
UNSURE_FRAC = 0.15


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


def check_g_bounds(g_gpu, g, g_lo, g_hi):
    """Slab overlap against the fp64 oracle under the marginal-decision rule;
    returns the number of pairs with a marginal decision."""
    fixed = g_lo == g_hi
    assert np.array_equal(g_gpu[fixed] == 0, g[fixed] == 0), "zero pattern differs"
    nz = fixed & (g != 0)
    assert np.all(np.abs(g_gpu[nz] / g[nz] - 1.0) <= G_RTOL), "g differs where the count is fixed"
    m = ~fixed
    assert np.all(g_gpu[m] >= g_lo[m] * (1 - G_RTOL)), "g below the marginal range"
    assert np.all(g_gpu[m] <= g_hi[m] * (1 + G_RTOL)), "g above the marginal range"
    n_marg = int(m.sum())
    assert n_marg <= max(2, MARGINAL_FRAC * g.size), f"{n_marg} marginal pairs"
    return n_marg


def check_coverage_bounds(rho_gpu, cov_gpu, n, n_lo, n_hi, b, eta):
    """Coverage against the fp64 oracle's counts under the marginal rule;
    returns the number of query blocks with a marginal token."""
    rho_gpu = np.asarray(rho_gpu)
    cnt = np.rint(rho_gpu.astype(np.float64) * b).astype(np.int64)
    assert np.array_equal(rho_gpu, (cnt / b).astype(np.float32)), "rho is not k / b"
    assert np.all((cnt >= n_lo) & (cnt <= n_hi)), "covered count outside the marginal range"
    fixed = n_lo == n_hi
    assert np.array_equal(cnt[fixed], n[fixed]), "covered count differs where it is fixed"
    assert np.array_equal(cov_gpu, (rho_gpu >= np.float32(eta)).astype(np.uint8))
    n_marg = int((~fixed).sum())
    assert n_marg <= max(2, MARGINAL_FRAC * len(n)), f"{n_marg} marginal blocks"
    return n_marg


def check_multiwarp(zq_gpu, zq_ref, unsure):
    """Multiwarp depths against the fp64 oracle; returns the unsure count."""
    sure = ~unsure
    assert np.array_equal(zq_gpu[sure] == 0, zq_ref[sure] == 0), "hole pattern differs"
    nz = sure & (zq_ref != 0)
    assert np.all(np.abs(zq_gpu[nz].astype(np.float64) / zq_ref[nz] - 1.0) <= MW_RTOL)
    n_uns = int(unsure.sum())
    assert n_uns <= max(2, UNSURE_FRAC * unsure.size), f"{n_uns} unsure tokens"
    return n_uns


def routes_from_gpu_p(layer, wl, g, covered, nbr):
    """Oracle routes of every (head, query block) row from the GPU's own p
    (the route step's input), compared with the GPU routes: bit-exact except
    at a mass cut within MASS_EPS of theta.  Returns ({(h, i): tile list},
    number of rows that differ at the cut)."""
    prm = oracle_params(wl.params)
    p = layer.p.cpu().numpy()
    g, cov = g.cpu().numpy(), covered.cpu().numpy()
    rid, rlen, rnb = layer.route_ids.cpu(), layer.route_len.cpu(), layer.route_nbudget.cpu()
    out, n_cut = {}, 0
    for h in range(wl.heads):
        for i in range(wl.n_q_blocks):
            ref = ort.route_row(p[h, i], g[i], bool(cov[i]), prm, wl.prev_begin,
                                wl.prev_count, list(nbr[i]))
            gpu = gpu_row(rid, rlen, rnb, h, i)
            n_cut += check_route_row(gpu, ref, f"head {h} row {i}") == "cut"
            out[(h, i)] = gpu[0] + gpu[1]
    return out, n_cut
