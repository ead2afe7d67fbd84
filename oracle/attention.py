"""Attention over routed 128-token KV tiles (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages' sparse attention (arXiv 2610.22311 digest, "Core method", Eq. 15;
Velox project page, "Why the route is a block, not a token") keeps or skips
whole KV tiles: query block i attends to every token of every tile in its
route R_i and to nothing else.  Its result is therefore exactly a softmax over
the tokens of the listed tiles, which this module computes directly in fp64
(no tiling, no online rescaling).

Readings: the softmax scale is 1/sqrt(d) unless given (standard scaled
dot-product attention; the pages are silent); there is no mask inside a tile;
a route is a set of tiles (a repeated id would be one tile); an empty route
gives O = 0 and lse = -inf.
"""

from __future__ import annotations

import math
from typing import Iterable, Tuple

import numpy as np


def routed_attention_block(q: np.ndarray, Kh: np.ndarray, Vh: np.ndarray,
                           tiles: Iterable[int], b: int,
                           scale: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """O and lse of one query block.

    q [b][d] (fp64), Kh and Vh [M*b][d] (fp64) of the same head; tiles are
    history block ids.  Returns (O [b][d], lse [b]) in fp64; lse is the
    natural-log normaliser log sum_t exp(scale * q . k_t).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[1]
    if scale <= 0.0:
        scale = 1.0 / math.sqrt(d)
    tiles = sorted(set(int(t) for t in tiles))
    if not tiles:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    idx = np.concatenate([np.arange(t * b, (t + 1) * b) for t in tiles])
    k = np.asarray(Kh[idx], dtype=np.float64)
    v = np.asarray(Vh[idx], dtype=np.float64)
    x = (q @ k.T) * scale
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    l = e.sum(axis=1, keepdims=True)
    O = (e @ v) / l
    lse = m[:, 0] + np.log(l[:, 0])
    return O, lse


def dense_attention_block(q, Kh, Vh, b: int, scale: float = 0.0):
    """Dense attention of one query block over all M history blocks."""
    M = Kh.shape[0] // b
    return routed_attention_block(q, Kh, Vh, range(M), b, scale)


def two_phase_attention_block(q: np.ndarray, Kh: np.ndarray, Vh: np.ndarray,
                              tiles: Iterable[int], Kc: np.ndarray, Vc: np.ndarray, b: int,
                              scale: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """Routed history tiles plus the current chunk's own keys, one softmax.

    The pages' kernel runs a "two-phase tile loop" (digest of arXiv
    2610.22311, "Reproducibility"): the routed history tiles of the KV cache
    and the tiles of the chunk being generated.  Reading: a query token
    attends to every token of its routed history tiles and to every token of
    the current chunk (Kc, Vc: [N_cur*b][d] of the same head), with one
    normaliser over both.  Returns (O [b][d], lse [b]) in fp64.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[1]
    if scale <= 0.0:
        scale = 1.0 / math.sqrt(d)
    tiles = sorted(set(int(t) for t in tiles))
    parts_k = [np.asarray(Kh[t * b:(t + 1) * b], dtype=np.float64) for t in tiles]
    parts_v = [np.asarray(Vh[t * b:(t + 1) * b], dtype=np.float64) for t in tiles]
    parts_k.append(np.asarray(Kc, dtype=np.float64))
    parts_v.append(np.asarray(Vc, dtype=np.float64))
    k = np.concatenate(parts_k)
    v = np.concatenate(parts_v)
    if k.shape[0] == 0:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    x = (q @ k.T) * scale
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    l = e.sum(axis=1, keepdims=True)
    return (e @ v) / l, m[:, 0] + np.log(l[:, 0])
