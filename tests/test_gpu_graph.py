"""The layer captured as a CUDA graph replays to the same bits as the eager
calls, also after new input values are copied into the captured tensors."""

import pytest
import torch

from routed_block_sparse_b200.pipeline import layer_for
from synth import config, make_inputs

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager(lib):
    wl = config(2)
    inp = make_inputs(wl, "cuda")
    layer = layer_for(wl)
    graph = layer.capture(inp.Q, inp.K, inp.V, inp.g, inp.covered)
    # eager reference on a second layer object with its own buffers
    ref = layer_for(wl)
    O_ref, lse_ref = ref.forward(inp.Q, inp.K, inp.V, inp.g, inp.covered)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.O, O_ref) and torch.equal(layer.lse, lse_ref)
    assert torch.equal(layer.route_ids, ref.route_ids)
    # new values in the same tensors: the replay follows them
    other = make_inputs(config(2).with_layer(1), "cuda")
    for dst, src in ((inp.Q, other.Q), (inp.K, other.K), (inp.V, other.V), (inp.g, other.g),
                     (inp.covered, other.covered)):
        dst.copy_(src)
    graph.replay()
    O2, lse2 = ref.forward(other.Q, other.K, other.V, other.g, other.covered)
    torch.cuda.synchronize()
    assert torch.equal(layer.O, O2) and torch.equal(layer.lse, lse2)
    assert layer.status() == 0
