"""Pins of the oracle's routed attention.

The routed result must equal a library scaled-dot-product attention (torch,
fp64, CPU) restricted by a boolean mask to the tokens of the listed tiles:
the pages' kernel keeps or skips whole tiles (Velox project page, "Why the
route is a block, not a token"; arXiv 2610.22311 digest, "Core method",
Eq. 15).  Also: the full route is dense attention, a single tile is textbook
softmax(q k^T / sqrt(d)) v, tile order and repeats do not matter, the
normaliser satisfies sum exp(x - lse) = 1, and an empty route gives zeros.
"""

import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import attention as at

B = 16
D = 32


def _data(seed, M):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, D))
    K = r.standard_normal((M * B, D))
    V = r.standard_normal((M * B, D))
    return q, K, V


def _sdpa(q, K, V, mask=None, scale=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None].expand(1, 1, q.shape[0], -1)
    out = F.scaled_dot_product_attention(t(q), t(K), t(V), attn_mask=m, scale=scale)
    return out[0, 0].numpy()


def test_routed_equals_masked_library_attention():
    M = 9
    q, K, V = _data(0, M)
    for tiles in ([3], [0, 8], [7, 2, 5], list(range(M))):
        mask = np.zeros(M * B, dtype=bool)
        for t in tiles:
            mask[t * B:(t + 1) * B] = True
        O, _ = at.routed_attention_block(q, K, V, tiles, B)
        assert np.allclose(O, _sdpa(q, K, V, mask), rtol=0, atol=1e-12)


def test_full_route_is_dense_and_scale_argument():
    q, K, V = _data(1, 6)
    O, _ = at.dense_attention_block(q, K, V, B)
    assert np.allclose(O, _sdpa(q, K, V), rtol=0, atol=1e-12)
    O2, _ = at.routed_attention_block(q, K, V, range(6), B, scale=0.3)
    assert np.allclose(O2, _sdpa(q, K, V, scale=0.3), rtol=0, atol=1e-12)


def test_single_tile_textbook():
    q, K, V = _data(2, 4)
    k, v = K[2 * B:3 * B], V[2 * B:3 * B]
    x = q @ k.T / math.sqrt(D)
    e = np.exp(x - x.max(axis=1, keepdims=True))
    want = (e / e.sum(axis=1, keepdims=True)) @ v
    O, _ = at.routed_attention_block(q, K, V, [2], B)
    assert np.allclose(O, want, rtol=0, atol=1e-13)


def test_order_repeats_and_lse():
    q, K, V = _data(3, 10)
    a, la = at.routed_attention_block(q, K, V, [1, 4, 9], B)
    b, lb = at.routed_attention_block(q, K, V, [9, 1, 4, 4, 1], B)
    assert np.allclose(a, b, rtol=0, atol=1e-14) and np.allclose(la, lb, rtol=0, atol=1e-14)
    idx = np.concatenate([np.arange(t * B, (t + 1) * B) for t in (1, 4, 9)])
    x = torch.from_numpy(q @ K[idx].T / math.sqrt(D))
    assert np.allclose(la, torch.logsumexp(x, dim=1).numpy(), rtol=0, atol=1e-12)
    assert np.allclose(np.exp(x.numpy() - la[:, None]).sum(axis=1), 1.0, atol=1e-12)


def test_empty_route():
    q, K, V = _data(4, 3)
    O, lse = at.routed_attention_block(q, K, V, [], B)
    assert np.all(O == 0) and np.all(np.isneginf(lse))


def test_two_phase_equals_library_attention_over_concatenated_keys():
    q, K, V = _data(5, 6)
    r = np.random.default_rng(5)
    Kc = r.standard_normal((3 * B, D))
    Vc = r.standard_normal((3 * B, D))
    tiles = [4, 1]
    O, lse = at.two_phase_attention_block(q, K, V, tiles, Kc, Vc, B)
    idx = np.concatenate([np.arange(t * B, (t + 1) * B) for t in sorted(tiles)])
    kk = np.concatenate([K[idx], Kc])
    vv = np.concatenate([V[idx], Vc])
    assert np.allclose(O, _sdpa(q, kk, vv), rtol=0, atol=1e-12)
    x = torch.from_numpy(q @ kk.T / math.sqrt(D))
    assert np.allclose(lse, torch.logsumexp(x, dim=1).numpy(), rtol=0, atol=1e-12)


def test_two_phase_is_the_merge_of_its_two_phases():
    # softmax over a union of disjoint key sets = the two partial results
    # merged with weights exp(lse_part - lse_all)
    q, K, V = _data(6, 7)
    r = np.random.default_rng(6)
    Kc = r.standard_normal((2 * B, D))
    Vc = r.standard_normal((2 * B, D))
    tiles = [0, 3, 6]
    Oh, lh = at.routed_attention_block(q, K, V, tiles, B)
    Oc, lc = at.routed_attention_block(q, Kc, Vc, [0, 1], B)
    O, lse = at.two_phase_attention_block(q, K, V, tiles, Kc, Vc, B)
    assert np.allclose(lse, np.logaddexp(lh, lc), rtol=0, atol=1e-12)
    want = np.exp(lh - lse)[:, None] * Oh + np.exp(lc - lse)[:, None] * Oc
    assert np.allclose(O, want, rtol=0, atol=1e-12)
    # no history tiles: plain attention over the current chunk
    O0, _ = at.two_phase_attention_block(q, K, V, [], Kc, Vc, B)
    assert np.allclose(O0, Oc, rtol=0, atol=1e-12)
