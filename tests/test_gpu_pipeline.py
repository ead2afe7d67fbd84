"""The whole path on the GPU (importance -> route -> attention) vs the oracle.

Every stage of the oracle runs on the oracle's own intermediate results, from
the same seeded inputs.  GPU routes must match the oracle's bit for bit except
at a mass cut that lies within fp32 reach of theta (the GPU importance is fp32);
attention is compared on rows whose routes match.
"""

import numpy as np
import pytest
import torch

from oracle import gilbert
from routed_block_sparse_b200.pipeline import layer_for
from synth import config, make_inputs, sweep_workload
from parity import (assert_attention_close, attention_rows, f64, gpu_row, oracle_importance,
                    oracle_params, oracle_routes, routes_from_gpu_p)

pytestmark = pytest.mark.gpu

# GPU p carries fp32 error (|dp/p| <= P_RTOL); scores this close to the cut
# may legitimately land on either side.
SCORE_BAND = 1e-4


def _compare(layer, inp, heads, attn_rows_per_head):
    wl = inp.wl
    torch.cuda.synchronize()
    assert layer.status() == 0
    p = oracle_importance(inp.Q, inp.K, heads)
    nbr = None
    if wl.lattice is not None:
        T, Hl, Wl = wl.lattice
        nbr = gilbert.neighbour_blocks(T, Hl, Wl, wl.n_chunks, 128, wl.q_chunk,
                                       wl.cache_first_block, wl.n_kv_blocks)
    ref = oracle_routes(p, inp.g.cpu().numpy(), inp.covered.cpu().numpy(),
                        oracle_params(wl.params), wl.prev_begin, wl.prev_count, nbr)
    rid, rlen, rnb = layer.route_ids.cpu(), layer.route_len.cpu(), layer.route_nbudget.cpu()
    same = []
    n_band = 0
    for (h, i), (budget, extras, info) in ref.items():
        gb, ge, _ = gpu_row(rid, rlen, rnb, h, i)
        if gb == budget and ge == extras:
            same.append((h, i))
            continue
        # allowed only inside the fp32 band around the cut score
        s, order, nw = info["s"], info["order"], info["n_walked"]
        cut = s[order[nw - 1]] if nw > 0 else s[order[0]]
        diff = set(gb) ^ set(budget)
        assert all(abs(s[x] - cut) <= SCORE_BAND * cut for x in diff), (h, i)
        n_band += 1
    assert n_band <= max(1, len(ref) // 50)
    rows = [r for r in same if r[1] in attn_rows_per_head]
    routes = {r: ref[r][0] + ref[r][1] for r in rows}
    oref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: routes[(h, i)])
    return assert_attention_close(layer.O, layer.lse, oref)


@pytest.mark.parametrize("cfg", [1, 2])
def test_pipeline_small_configs(lib, cfg):
    wl = config(cfg)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
    _compare(layer, inp, range(wl.heads), range(wl.n_q_blocks) if cfg == 1 else (0, 5, 11))


@pytest.mark.slow
def test_pipeline_chunk48(lib):
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
    _compare(layer, inp, [0, 39], (0, 23, 47))


@pytest.mark.slow
def test_pipeline_sweep_and_dense(lib):
    for M in (64, 1024, 4096):
        wl = sweep_workload(M)
        inp = make_inputs(wl, "cuda")
        layer = layer_for(wl)
        layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
        _compare(layer, inp, [7], (1, 40))
        O, lse = layer.attend(inp.Q, inp.K, inp.V, dense=True)
        torch.cuda.synchronize()
        rows = [(3, 0), (38, 47)]
        ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: range(M))
        assert_attention_close(O, lse, ref)
        del inp, layer
        torch.cuda.empty_cache()


@pytest.mark.slow
def test_pipeline_forty_layers(lib):
    """The 40-layer workload (per-layer seeds, regenerated into reused
    buffers): route sets of every head and query block of all 40 layers,
    importance on 4 heads of every layer, attention on 4 heads x 8 rows of
    layers 0 and 39."""
    wl0 = config(5, 0)
    layer = layer_for(wl0)
    inp = make_inputs(wl0, "cuda")
    T, Hl, Wl = wl0.lattice
    nbr = gilbert.neighbour_blocks(T, Hl, Wl, wl0.n_chunks, 128, wl0.q_chunk,
                                   wl0.cache_first_block, wl0.n_kv_blocks)
    from parity import P_RTOL
    for li in range(40):
        wl = config(5, li)
        inp = make_inputs(wl, "cuda", out=inp)
        layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
        torch.cuda.synchronize()
        assert layer.status() == 0, f"layer {li}"
        routes, n_cut = routes_from_gpu_p(layer, wl, inp.g, inp.covered, nbr)
        assert n_cut <= 2, f"layer {li}: {n_cut} rows differ at the cut"
        heads = [(li + 10 * k) % 40 for k in range(4)]
        for h, ph in oracle_importance(inp.Q, inp.K, heads).items():
            rel = np.abs(f64(layer.p[h]) / ph - 1.0).max()
            assert rel <= P_RTOL, f"layer {li} head {h}: importance rel err {rel}"
        if li in (0, 39):
            rng = np.random.default_rng(li)
            rows = [(h, int(i)) for h in heads for i in rng.choice(48, size=8, replace=False)]
            ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: routes[(h, i)])
            assert_attention_close(layer.O, layer.lse, ref)


@pytest.mark.slow
def test_chunk48_attention_rows_of_every_wave(lib):
    """The bench's launch (longest-route-first row order, one CTA per SM):
    one row from each wave of that order, the last row of the final wave and
    its neighbours, against the oracle on the layer's own routes."""
    wl = config(3)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
    torch.cuda.synchronize()
    assert layer.status() == 0
    order = layer.row_order.cpu().numpy()
    lens = layer.route_len.cpu().numpy().reshape(-1)
    assert np.all(np.diff(lens[order]) <= 0)       # longest first
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows_total = len(order)
    pos = sorted(set(list(range(0, rows_total, sms)) + [rows_total - 3, rows_total - 2,
                                                        rows_total - 1]))
    N = wl.n_q_blocks
    rows = sorted({(int(order[k]) // N, int(order[k]) % N) for k in pos})
    rid, rlen = layer.route_ids.cpu(), layer.route_len.cpu()
    routes = {(h, i): rid[h, i, :int(rlen[h, i])].tolist() for (h, i) in rows}
    ref = attention_rows(inp.Q, inp.K, inp.V, rows, lambda h, i: routes[(h, i)])
    assert_attention_close(layer.O, layer.lse, ref)
