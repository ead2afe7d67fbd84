"""Calls from several host threads on their own streams (the header's
re-entrancy claim): two threads each run whole layers, concurrently, and
every output equals the one the same layer gives when run alone."""

import threading
from dataclasses import replace

import pytest
import torch

from routed_block_sparse_b200.pipeline import layer_for
from synth import config, make_inputs

pytestmark = pytest.mark.gpu


def test_two_threads_two_streams_same_bits(lib):
    wls = [replace(config(3, layer), heads=4) for layer in (0, 1, 2, 3)]
    inps = [make_inputs(wl, "cuda") for wl in wls]
    # alone, one after the other
    alone = []
    for wl, inp in zip(wls, inps):
        layer = layer_for(wl)
        O, lse = layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
        torch.cuda.synchronize()
        alone.append((O.clone(), lse.clone(), layer.route_ids.clone(), layer.status()))
    # two threads, each with its own stream and layers, three rounds each
    results = {}
    errors = []

    def worker(t):
        try:
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                for rnd in range(3):
                    for k in (t, t + 2):
                        layer = layer_for(wls[k])
                        inp = inps[k]
                        layer.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered, stream)
                        stream.synchronize()
                        results[(t, rnd, k)] = (layer.O.clone(), layer.lse.clone(),
                                                layer.route_ids.clone(), layer.status())
        except Exception as e:  # reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(t,)) for t in (0, 1)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=300)
    torch.cuda.synchronize()
    assert not errors, errors
    assert len(results) == 12
    for (t, rnd, k), (O, lse, rid, st) in results.items():
        a = alone[k]
        assert st == 0 and a[3] == 0
        assert torch.equal(rid, a[2]), (t, rnd, k)
        assert torch.equal(O, a[0]) and torch.equal(lse, a[1]), (t, rnd, k)
