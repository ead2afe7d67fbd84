"""GPU block importance vs the oracle (fp32 vs fp64, relative tolerance)."""

import math

import numpy as np
import pytest
import torch

from synth import config, make_inputs
from synth.configs import small
from parity import P_RTOL, f64, oracle_importance

pytestmark = pytest.mark.gpu


def _run(lib, inp, scale):
    wl = inp.wl
    H, N, M = wl.heads, wl.n_q_blocks, wl.n_kv_blocks
    p = torch.full((H, N, M), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.velox_workspace_size(H, N, M), dtype=torch.uint8, device="cuda")
    lib.velox_block_importance(inp.Q, inp.K, H, N, M, 128, 128, scale, p, ws)
    torch.cuda.synchronize()
    return p


def _check(p, ref):
    for h, ph in ref.items():
        g = f64(p[h])
        assert np.all(np.isfinite(g))
        rel = np.abs(g / ph - 1.0).max()
        assert rel <= P_RTOL, f"head {h}: rel err {rel}"
        assert abs(g.sum(axis=1) - 1.0).max() < 1e-4


@pytest.mark.parametrize("cfg", [1, 2])
@pytest.mark.parametrize("scale", [1.0, 1.0 / math.sqrt(128)])
def test_importance_small_configs(lib, cfg, scale):
    inp = make_inputs(config(cfg), "cuda")
    p = _run(lib, inp, scale)
    _check(p, oracle_importance(inp.Q, inp.K, range(inp.wl.heads), scale))


@pytest.mark.slow
def test_importance_chunk48_every_head(lib):
    # the bench's launch: 40 heads, chunks that start anywhere in a head's
    # 2256 key blocks; every head against the oracle
    inp = make_inputs(config(3), "cuda")
    p = _run(lib, inp, 1.0)
    _check(p, oracle_importance(inp.Q, inp.K, range(inp.wl.heads), 1.0))


@pytest.mark.parametrize("H,N,M", [(1, 1, 1), (2, 3, 65), (3, 17, 130), (1, 40, 200),
                                   (1, 2, 1024), (1, 2, 1028), (2, 3, 2304), (1, 2, 2308),
                                   (2, 3, 4096)])
def test_importance_ragged_shapes(lib, H, N, M):
    # M = 1024 / 2304 / 4096 are the largest rows of each register-resident
    # softmax width (8, 18, 32 float4 per lane), 1028 and 2308 the smallest
    # above them; M not a multiple of 4 takes the CTA-per-row softmax
    inp = make_inputs(small(H, N, M, 0), "cuda")
    p = _run(lib, inp, 1.0)
    _check(p, oracle_importance(inp.Q, inp.K, range(H), 1.0))


@pytest.mark.parametrize("H,M", [(1, 300), (8, 300), (16, 300), (24, 300), (32, 300),
                                 (39, 300), (19, 777), (17, 1000)])
def test_importance_every_chunk_width(lib, H, M):
    # The fused kernel streams chunks of 8 * w key blocks (w per warp, 1..8,
    # picked from H and M).  On a 148-SM part with two CTAs per SM these
    # shapes pick w = 1, 2, ..., 8 in turn, and each ends on a partial chunk
    # (warps with fewer than w blocks and warps with none).  N = 5 is odd.
    inp = make_inputs(small(H, 5, M, 0), "cuda")
    p = _run(lib, inp, 1.0)
    _check(p, oracle_importance(inp.Q, inp.K, range(H), 1.0))


def test_importance_peaked_logits(lib):
    # large scale: logits of order 100, rows nearly one-hot.  An fp32 logit
    # carries an absolute error of about |logit| * 2^-23 ~ 1e-5, which turns
    # into the same relative error of p: bound it at 50 * P_RTOL (1e-3).
    inp = make_inputs(small(2, 4, 50, 0, key_mean_sigma=2.0), "cuda")
    p = _run(lib, inp, 8.0)
    ref = oracle_importance(inp.Q, inp.K, range(2), 8.0)
    for h, ph in ref.items():
        g = f64(p[h])
        assert np.all(np.abs(g - ph) <= 50 * P_RTOL * ph + 1e-30)


def test_importance_at_the_largest_history(lib):
    # M = VELOX_MAX_BLOCKS (65536): p of one row, checked where the oracle
    # can afford it -- the row sums to 1, and sampled pairs of blocks have
    # the fp64 ratio p_r / p_s = exp(l_r - l_s) of their own mean keys
    H, N, M = 1, 1, 65536
    inp = make_inputs(small(H, N, M, 0), "cuda")
    p = f64(_run(lib, inp, 1.0)[0, 0])
    assert np.all(np.isfinite(p)) and abs(p.sum() - 1.0) < 1e-4
    qbar = f64(inp.Q[0, :128]).mean(axis=0)
    r = np.random.default_rng(5)
    ids = r.choice(M, size=24, replace=False)
    kbar = {int(b): f64(inp.K[0, b * 128:(b + 1) * 128]).mean(axis=0) for b in ids}
    for a_, b_ in zip(ids[::2], ids[1::2]):
        ratio = math.exp(float(qbar @ kbar[int(a_)] - qbar @ kbar[int(b_)]))
        assert abs(p[a_] / p[b_] / ratio - 1.0) <= 2 * P_RTOL
