"""Per-head block importance (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages define the layer's own block importance p_{i,r} as a softmax over
history blocks r of the inner product of the mean query of query block i and
the mean key of history block r (arXiv 2610.22311 digest, "Method steps", step
four, Eq. 9; onedev.kr summary, "How it differs"; Velox project page,
"02 · Method", glossary entry for p).

Readings: the product is multiplied by ``scale`` before the softmax (the pages
give no temperature; 1.0 is the default, 1/sqrt(d) is the model-faithful
alternative); the softmax runs over all M cache blocks, reserved ones included.

Inputs are one head at a time, as float64 arrays holding the exact bf16 values.
"""

from __future__ import annotations

import numpy as np


def block_means(X: np.ndarray, b: int) -> np.ndarray:
    """Mean over each run of b consecutive tokens: [n*b][d] -> [n][d] (fp64)."""
    L, d = X.shape
    if L % b != 0:
        raise ValueError("token count not a multiple of the block size")
    return X.reshape(L // b, b, d).mean(axis=1, dtype=np.float64)


def importance(Qh: np.ndarray, Kh: np.ndarray, b: int, scale: float) -> np.ndarray:
    """p[i, r] = softmax_r(scale * qbar_i . kbar_r) for one head: [N][M] fp64."""
    qbar = block_means(np.asarray(Qh, dtype=np.float64), b)
    kbar = block_means(np.asarray(Kh, dtype=np.float64), b)
    logits = float(scale) * (qbar @ kbar.T)
    logits = logits - logits.max(axis=1, keepdims=True)
    e = np.exp(logits)
    return e / e.sum(axis=1, keepdims=True)
