"""velox_block_importance_noalloc against velox_block_importance.

The no-allocation variant exists for callers that cannot allocate device
memory (a framework that budgets all GPU memory up front and gives plugins no
allocator, or a loop that cannot take cudaMalloc's device-wide
synchronisation).  It keeps the block means in a fixed array inside the
library instead of a caller workspace, so its results must match the
workspace entry point's within the importance tolerance of the other tests,
on consecutive calls that reuse (and inherit the contents of) that array.

This file is collected last on purpose: it must pass both alone in a fresh
process and after every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from parity import P_RTOL, f64, oracle_importance
from synth.configs import small
from synth import config, make_inputs

pytestmark = pytest.mark.gpu


def _with_workspace(rbs, inp):
    wl = inp.wl
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    p = torch.empty(H, N, M, dtype=torch.float32, device="cuda")
    ws = torch.empty(rbs.velox_workspace_size(H, N, M), dtype=torch.uint8, device="cuda")
    rbs.velox_block_importance(inp.Q, inp.K, H, N, M, 128, 128, 1.0, p, ws)
    return p


def _no_alloc(rbs, inp):
    wl = inp.wl
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    p = torch.full((H, N, M), float("nan"), dtype=torch.float32, device="cuda")
    rbs.velox_block_importance_noalloc(inp.Q, inp.K, H, N, M, 128, 128, 1.0, p)
    return p


def test_no_alloc_matches_workspace_entry_on_consecutive_calls():
    import routed_block_sparse_b200 as rbs
    # calls in a row on different shapes: each call inherits the previous
    # call's leftovers in the shared array and must not depend on them.  The
    # first case has N > 96 query blocks, so its key means go through the
    # array (the unfused path) and the fused calls after it find key means
    # left behind there.
    cases = [make_inputs(small(2, 100, 300, 0), "cuda"), make_inputs(config(2), "cuda"),
             make_inputs(small(3, 5, 301, 0), "cuda")]
    for inp in cases:
        ref = _with_workspace(rbs, inp)
        got = _no_alloc(rbs, inp)
        torch.cuda.synchronize()
        g, r = f64(got), f64(ref)
        assert np.all(np.isfinite(g))
        assert np.all(np.abs(g - r) <= P_RTOL * np.abs(r)), "no-alloc importance differs"
        # and against the oracle's definition, on up to three heads
        heads = range(min(3, inp.wl.heads))
        for h, ph in oracle_importance(inp.Q, inp.K, heads, 1.0).items():
            assert np.abs(g[h] / ph - 1.0).max() <= P_RTOL, f"head {h} vs oracle"


def test_no_alloc_rejects_sizes_beyond_its_array():
    import routed_block_sparse_b200 as rbs
    # H * (N + M) * 128 * 4 bytes must fit in the fixed array
    H, N = 40, 48
    M = rbs.NOALLOC_SCRATCH_BYTES // (H * 128 * 4) - N + 1
    Q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    p = torch.empty(16, dtype=torch.float32, device="cuda")
    # the library refuses the sizes before launching (called through the C
    # entry point: the tensors here are far smaller than the sizes say)
    P = ctypes.c_void_p
    st = rbs._lib.velox_block_importance_noalloc(P(Q.data_ptr()), P(Q.data_ptr()), H, N, M, 128,
                                                 128, 1.0, P(p.data_ptr()), None)
    assert st == 3  # VELOX_ERR_WORKSPACE, nothing launched
    # and the binding refuses the undersized tensors before the call
    with pytest.raises(ValueError):
        rbs.velox_block_importance_noalloc(Q, Q, H, N, M, 128, 128, 1.0, p)
