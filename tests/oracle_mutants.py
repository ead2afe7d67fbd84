"""Planted mistakes in the oracle, to show that its pins pin (test
infrastructure only).

Each entry changes one line of one oracle module in a plausible way: a
dropped term, a flipped sign or comparison, a swapped index or operand, an
off-by-one.  tests/test_oracle_mutants.py runs the module's own pin file in
a child pytest process with the change applied (through the environment
variable VELOX_ORACLE_MUTANT, read by conftest.py) and requires that some pin
fails.  The mistakes are planted on the CPU, in the oracle, never in the CUDA
path.

Entry: (name, oracle module, exact text, replacement, pin test file).

Not listed because no pin can tell them apart from the oracle: changes of the
Gilbert construction's split rule (for example a two-way split whenever the
major edge is longer) that still give a unit-step curve from (0, 0) to
(W-1, 0); the exact curve beyond its invariants is unpinned against the
authors' figures, whose ranks are not in the text.
"""

from __future__ import annotations

import importlib
import inspect

MUTANTS = [
    # ---- block importance
    ("importance: scale dropped", "oracle.importance",
     "logits = float(scale) * (qbar @ kbar.T)", "logits = (qbar @ kbar.T)",
     "test_oracle_importance.py"),
    ("importance: block sums instead of means", "oracle.importance",
     "return X.reshape(L // b, b, d).mean(axis=1, dtype=np.float64)",
     "return X.reshape(L // b, b, d).sum(axis=1, dtype=np.float64)",
     "test_oracle_importance.py"),
    ("importance: normalised over query blocks", "oracle.importance",
     "return e / e.sum(axis=1, keepdims=True)", "return e / e.sum(axis=0, keepdims=True)",
     "test_oracle_importance.py"),
    ("importance: max subtracted per column", "oracle.importance",
     "logits = logits - logits.max(axis=1, keepdims=True)",
     "logits = logits - logits.max(axis=0, keepdims=True)",
     "test_oracle_importance.py"),
    ("importance: token and channel axes swapped", "oracle.importance",
     "return X.reshape(L // b, b, d).mean(axis=1, dtype=np.float64)",
     "return X.reshape(L // b, d, b).mean(axis=2, dtype=np.float64)",
     "test_oracle_importance.py"),
    # ---- attention
    ("attention: scale 1/d", "oracle.attention",
     """    if scale <= 0.0:
        scale = 1.0 / math.sqrt(d)
    tiles = sorted(set(int(t) for t in tiles))
    if not tiles:""",
     """    if scale <= 0.0:
        scale = 1.0 / d
    tiles = sorted(set(int(t) for t in tiles))
    if not tiles:""",
     "test_oracle_attention.py"),
    ("attention: lse without the max", "oracle.attention",
     "lse = m[:, 0] + np.log(l[:, 0])", "lse = np.log(l[:, 0])",
     "test_oracle_attention.py"),
    ("attention: keys as values", "oracle.attention",
     "O = (e @ v) / l", "O = (e @ k) / l", "test_oracle_attention.py"),
    ("attention: last token of each tile dropped", "oracle.attention",
     "np.arange(t * b, (t + 1) * b) for t in tiles", "np.arange(t * b, (t + 1) * b - 1) for t in tiles",
     "test_oracle_attention.py"),
    ("attention: repeated tile counted twice", "oracle.attention",
     """    tiles = sorted(set(int(t) for t in tiles))
    if not tiles:""",
     """    tiles = sorted(int(t) for t in tiles)
    if not tiles:""",
     "test_oracle_attention.py"),
    ("two-phase: current keys as current values", "oracle.attention",
     "parts_v.append(np.asarray(Vc, dtype=np.float64))",
     "parts_v.append(np.asarray(Kc, dtype=np.float64))", "test_oracle_attention.py"),
    ("two-phase: separate normalisers", "oracle.attention",
     "    return (e @ v) / l, m[:, 0] + np.log(l[:, 0])",
     "    nh = sum(len(p) for p in parts_v[:-1])\n"
     "    lh = e[:, :nh].sum(axis=1, keepdims=True) + (nh == 0)\n"
     "    lc = e[:, nh:].sum(axis=1, keepdims=True)\n"
     "    return (e[:, :nh] @ v[:nh]) / lh + (e[:, nh:] @ v[nh:]) / lc, m[:, 0] + np.log(l[:, 0])",
     "test_oracle_attention.py"),
    # ---- fusion and route
    ("route: g >= tau", "oracle.route",
     "ghat = np.where(g > _f32(prm.tau),", "ghat = np.where(g >= _f32(prm.tau),",
     "test_oracle_route.py"),
    ("route: ghat cap dropped", "oracle.route",
     "np.minimum(g / _f32(prm.g_ref), 1.0)", "g / _f32(prm.g_ref)", "test_oracle_route.py"),
    ("route: fusion sign flipped", "oracle.route",
     "return p * (1.0 + _f32(prm.lam) * ghat)", "return p * (1.0 - 0.25 * _f32(prm.lam) * ghat)",
     "test_oracle_route.py"),
    ("route: covered rows not renormalised", "oracle.route",
     "s = key / key.sum()", "s = key", "test_oracle_route.py"),
    ("route: cut at mass > theta", "oracle.route",
     "if len(budget) >= K or mass >= theta:", "if len(budget) >= K or mass > theta:",
     "test_oracle_route.py"),
    ("route: reserved blocks outside the count", "oracle.route",
     "if len(budget) >= K or mass >= theta:",
     "if len(budget) - len(reserved) >= K or mass >= theta:", "test_oracle_route.py"),
    ("route: reserved mass ignored", "oracle.route",
     """    for r in reserved:
        mass += s[r]""",
     """    for r in reserved:
        mass += 0.0""", "test_oracle_route.py"),
    ("route: ties to the higher id", "oracle.route",
     "rest = rest[np.lexsort((rest, -key[rest]))]", "rest = rest[np.lexsort((-rest, -key[rest]))]",
     "test_oracle_route.py"),
    ("route: extras not deduplicated against the budget", "oracle.route",
     "extras = sorted(set(int(u) for u in safeguards) - bset)",
     "extras = sorted(set(int(u) for u in safeguards))", "test_oracle_route.py"),
    ("route: covered rows sorted by the model's p", "oracle.route",
     """        key = fused_weight(p_row, g_row, prm)
        s = key / key.sum()""",
     """        key = fused_weight(p_row, g_row, prm)
        s = key / key.sum()
        key = p""", "test_oracle_route.py"),
    ("route: uncovered rows fused too", "oracle.route",
     """        key = p
        s = p
        K, theta = prm.k_unc, _f32(prm.theta_unc)""",
     """        key = fused_weight(p_row, g_row, prm)
        s = key / key.sum()
        K, theta = prm.k_unc, _f32(prm.theta_unc)""", "test_oracle_route.py"),
    ("route: covered rows use the uncovered cap", "oracle.route",
     "K, theta = prm.k_cov, _f32(prm.theta_cov)", "K, theta = prm.k_unc, _f32(prm.theta_cov)",
     "test_oracle_route.py"),
    # ---- Gilbert order and neighbours
    ("gilbert: no mirror on odd frames", "oracle.gilbert",
     "frame = r2[:, ::-1] if f % 2 == 1 else r2", "frame = r2", "test_oracle_gilbert.py"),
    ("gilbert: mirror on even frames", "oracle.gilbert",
     "frame = r2[:, ::-1] if f % 2 == 1 else r2", "frame = r2[:, ::-1] if f % 2 == 0 else r2",
     "test_oracle_gilbert.py"),
    ("gilbert: block ids from the inverse map", "oracle.gilbert",
     """    cell_of_rank[rank_of_cell] = np.arange(rank_of_cell.size)
    return rank_of_cell, cell_of_rank, rank_of_cell // b


def thw_linear_order""",
     """    cell_of_rank[rank_of_cell] = np.arange(rank_of_cell.size)
    return rank_of_cell, cell_of_rank, cell_of_rank // b


def thw_linear_order""", "test_oracle_gilbert.py"),
    ("gilbert: halves not made even", "oracle.gilbert",
     "if abs(hax + hay) % 2 == 1 and n_major > 2:", "if False:", "test_oracle_gilbert.py"),
    ("gilbert: far piece not mirrored back", "oracle.gilbert",
     "-hbx, -hby, -(ax - hax), -(ay - hay))", "hbx, hby, -(ax - hax), -(ay - hay))",
     "test_oracle_gilbert.py"),
    ("neighbours: no look back in time", "oracle.gilbert",
     "for df in (-1, 0, 1):", "for df in (0, 1):", "test_oracle_gilbert.py"),
    ("neighbours: own block kept", "oracle.gilbert",
     "if u != qb and lo <= u < hi:", "if lo <= u < hi:", "test_oracle_gilbert.py"),
    ("thw: column-major frames", "oracle.gilbert",
     "rank[f, y, x] = (f * H + y) * W + x", "rank[f, y, x] = (f * W + x) * H + y",
     "test_oracle_gilbert.py"),
    # ---- slab overlap and coverage
    ("geometry: full extents as half extents", "oracle.geometry",
     "half = np.array([(u1 - u0) / (2.0 * fx) * zm,", "half = np.array([(u1 - u0) / fx * zm,",
     "test_oracle_geometry.py"),
    ("geometry: union without the intersection", "oracle.geometry",
     "union = vi + vr - inter", "union = vi + vr", "test_oracle_geometry.py"),
    ("geometry: box frame with R instead of R^T", "oracle.geometry",
     "d = (X - cr) @ Rr                      # box-frame", "d = (X - cr) @ Rr.T                    # box-frame",
     "test_oracle_geometry.py"),
    ("geometry: grid at cell corners", "oracle.geometry",
     "s = (2.0 * np.arange(G) + 1.0) / G - 1.0", "s = (2.0 * np.arange(G)) / G - 1.0",
     "test_oracle_geometry.py"),
    ("geometry: token unprojection multiplies by f", "oracle.geometry",
     "return C + R @ np.array([(u - cx) / fx * z, (v - cy) / fy * z, z])",
     "return C + R @ np.array([(u - cx) * fx * z, (v - cy) / fy * z, z])",
     "test_oracle_geometry.py"),
    ("geometry: rectangle closed on the right", "oracle.geometry",
     "in_u = (u0 <= pu) & (pu < u1)", "in_u = (u0 <= pu) & (pu <= u1)", "test_oracle_geometry.py"),
    ("geometry: depth interval open", "oracle.geometry",
     "in_z = (zlo <= pz) & (pz <= zhi)", "in_z = (zlo < pz) & (pz < zhi)", "test_oracle_geometry.py"),
    ("geometry: covered at rho > eta", "oracle.geometry",
     "return rho, (rho >= float(np.float32(eta))).astype(np.uint8)",
     "return rho, (rho > float(np.float32(eta))).astype(np.uint8)", "test_oracle_geometry.py"),
    # ---- slab table, block tokens, multiwarp
    ("slabs: percentile at n q", "oracle.slabs",
     "h = (n - 1) * q", "h = n * q if n * q <= n - 1 else n - 1", "test_oracle_slabs.py"),
    ("slabs: rectangle right edge inclusive", "oracle.slabs",
     "slab[j] = [min(xs), max(xs) + 1, min(ys), max(ys) + 1,",
     "slab[j] = [min(xs), max(xs), min(ys), max(ys) + 1,", "test_oracle_slabs.py"),
    ("slabs: confidence filter dropped", "oracle.slabs",
     "ok = ok and (conf is None or float(conf[lf, py, px]) >= float(F(prm.c_min)))",
     "ok = ok", "test_oracle_slabs.py"),
    ("slabs: minimum sample count off by one", "oracle.slabs",
     "if len(samples) < prm.n_min or not samples:", "if len(samples) <= prm.n_min or not samples:",
     "test_oracle_slabs.py"),
    ("block tokens: x and y swapped", "oracle.slabs",
     "            y, x = divmod(rem, W)\n            z = float(depth[f - frame_base, y, x])",
     "            x, y = divmod(rem, W)\n            z = float(depth[f - frame_base, y, x])",
     "test_oracle_slabs.py"),
    ("block tokens: corner instead of centre", "oracle.slabs",
     "out[j, t] = [x + 0.5, y + 0.5, z if ok else 0.0]", "out[j, t] = [x, y, z if ok else 0.0]",
     "test_oracle_slabs.py"),
    ("block tokens: confidence filter dropped", "oracle.slabs",
     "            ok = ok and (conf is None or float(conf[f - frame_base, y, x]) >= float(F(c_min)))\n",
     "", "test_oracle_slabs.py"),
    ("multiwarp: landing by rounding", "oracle.slabs",
     "return (math.floor(pu), math.floor(pv)), pz, margin, cand",
     "return (int(round(pu)), int(round(pv))), pz, margin, cand", "test_oracle_slabs.py"),
    ("multiwarp: oldest source first", "oracle.slabs",
     "            for got in per_src:\n", "            for got in per_src[::-1]:\n",
     "test_oracle_slabs.py"),
    ("multiwarp: k_warp exceeded instead of reached", "oracle.slabs",
     "if len(vals) >= k_warp:", "if len(vals) > k_warp:", "test_oracle_slabs.py"),
    ("multiwarp: sample at its corner", "oracle.slabs",
     "                u = (px + 0.5) / s\n                v = (py + 0.5) / s",
     "                u = px / s\n                v = py / s", "test_oracle_slabs.py"),
    # ---- audit
    ("audit: g >= tau positive", "oracle.audit",
     "pos = {r for r in range(len(p)) if g[r] > float(np.float32(prm.tau))}",
     "pos = {r for r in range(len(p)) if g[r] >= float(np.float32(prm.tau))}",
     "test_oracle_audit.py"),
    ("audit: R_50 over M", "oracle.audit",
     "R_50=c[2] / (rows * min(k_geo, M)),", "R_50=c[2] / (rows * M),", "test_oracle_audit.py"),
    ("audit: ties to the higher id", "oracle.audit",
     "order = sorted(range(M), key=lambda r: (-float(score[r]), r))",
     "order = sorted(range(M), key=lambda r: (-float(score[r]), -r))", "test_oracle_audit.py"),
    ("audit: recall against the geometry's own top-K", "oracle.audit",
     "len(pos & a_geo), len(g_geo & a_geo)", "len(pos & g_geo), len(g_geo & a_geo)",
     "test_oracle_audit.py"),
    # ---- marginal-decision bounds (the GPU parity rule's ranges)
    ("geometry: marginal lower count includes the face band", "oracle.geometry",
     "n_lo = int(np.count_nonzero(margin > eps))", "n_lo = int(np.count_nonzero(margin >= -eps))",
     "test_oracle_geometry.py"),
    ("geometry: marginal upper count drops the face band", "oracle.geometry",
     "n_hi = int(np.count_nonzero(margin >= -eps))", "n_hi = int(np.count_nonzero(margin > eps))",
     "test_oracle_geometry.py"),
    ("geometry: coverage upper count ignores near misses", "oracle.geometry",
     "n_hi[i] += bool((inside | (margin <= eps)).any())", "n_hi[i] += bool(inside.any())",
     "test_oracle_geometry.py"),
    ("geometry: inside margin takes the farthest face", "oracle.geometry",
     "m_in = np.minimum(np.minimum(du, dv), dz)", "m_in = np.maximum(np.maximum(du, dv), dz)",
     "test_oracle_geometry.py"),
    ("multiwarp: marginal landings not marked unsure", "oracle.slabs",
     "                if margin <= eps:\n                    for (x, y) in cand:",
     "                if margin < -1.0:\n                    for (x, y) in cand:",
     "test_oracle_slabs.py"),
    ("multiwarp: candidates only the landing cell", "oracle.slabs",
     "xs = {math.floor(pu - du), math.floor(pu), math.floor(pu + du)}", "xs = {math.floor(pu)}",
     "test_oracle_slabs.py"),
    ("multiwarp: median of the first two samples", "oracle.slabs",
     "zq[y, x] = np.float32(np.median(np.asarray(vals, dtype=np.float64)))",
     "zq[y, x] = np.float32(np.mean(np.asarray(vals[:2], dtype=np.float64)))",
     "test_oracle_slabs.py"),
    # ---- audit pooling
    ("audit: R_geo averaged per row", "oracle.audit",
     "R_geo=c[1] / n_pos if n_pos else float(\"nan\"),",
     "R_geo=float(np.nanmean(np.asarray(counts).reshape(-1, 6)[:, 1] / np.maximum(np.asarray(counts).reshape(-1, 6)[:, 0], 1))),",
     "test_oracle_audit.py"),
    ("audit: changed counted against the model's top-50", "oracle.audit",
     "len(pos & f_fuse), len(f_fuse - a_fuse)", "len(pos & f_fuse), len(f_fuse - a_geo)",
     "test_oracle_audit.py"),
    # ---- Gilbert construction details
    ("gilbert: minor halves not made even", "oracle.gilbert",
     "if abs(hbx + hby) % 2 == 1 and n_minor > 2:", "if False:", "test_oracle_gilbert.py"),
    ("thw: neighbours from the Gilbert blocks", "oracle.gilbert",
     'order = {"gilbert": global_order, "thw": thw_linear_order}[layout]',
     'order = {"gilbert": global_order, "thw": global_order}[layout]', "test_oracle_gilbert.py"),
    # ---- importance / route details
    ("route: reserved range off by one", "oracle.route",
     "reserved = list(range(prev_begin, prev_begin + prev_count))",
     "reserved = list(range(prev_begin, prev_begin + prev_count - 1))", "test_oracle_route.py"),
    ("route: budget left unsorted", "oracle.route",
     "return sorted(budget), extras, info", "return budget, extras, info", "test_oracle_route.py"),
    ("attention: scale applied after the max", "oracle.attention",
     """    x = (q @ k.T) * scale
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    l = e.sum(axis=1, keepdims=True)
    O = (e @ v) / l""",
     """    x = (q @ k.T)
    m = x.max(axis=1, keepdims=True)
    e = np.exp((x - m) * scale)
    l = e.sum(axis=1, keepdims=True)
    O = (e @ v) / l""", "test_oracle_attention.py"),
]


def apply_mutant(k: int) -> None:
    """Re-executes the oracle module of entry k with its one change, in the
    module's own namespace (so every reference to the module sees it)."""
    name, modname, old, new, _ = MUTANTS[k]
    mod = importlib.import_module(modname)
    src = inspect.getsource(mod)
    if src.count(old) != 1:
        raise RuntimeError(f"mutant {name!r}: text found {src.count(old)} times")
    exec(compile(src.replace(old, new), mod.__file__, "exec"), mod.__dict__)
