"""Pins of the oracle's block importance (softmax of mean query . mean key).

Checked against closed forms and invariants that the definition fixes
(arXiv 2610.22311 digest, "Method steps", Eq. 9; onedev.kr summary, "How it
differs"): a two-block logistic closed form, rows summing to one, uniform rows
for equal keys, invariance to a shift shared by all keys, invariance to the
order of tokens inside a block, equivariance under block permutations, and a
mean taken over tokens (not over channels).
"""

import math

import numpy as np

from oracle import importance as imp

B = 8
D = 16


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_rows_sum_to_one_and_positive():
    r = _rng(1)
    Q = r.standard_normal((3 * B, D))
    K = r.standard_normal((11 * B, D))
    p = imp.importance(Q, K, B, 1.0)
    assert p.shape == (3, 11)
    assert np.all(p > 0)
    assert np.all(np.abs(p.sum(axis=1) - 1.0) < 1e-12)


def test_two_block_logistic_closed_form():
    # Constant tokens inside each block: the means are the constants, and with
    # two history blocks p_0 = 1 / (1 + exp(s q.(a1 - a0))).
    r = _rng(2)
    q = r.standard_normal(D)
    a0, a1 = r.standard_normal(D), r.standard_normal(D)
    Q = np.tile(q, (B, 1))
    K = np.concatenate([np.tile(a0, (B, 1)), np.tile(a1, (B, 1))])
    for s in (1.0, 0.25, 3.0):
        p = imp.importance(Q, K, B, s)
        want0 = 1.0 / (1.0 + math.exp(s * float(q @ (a1 - a0))))
        assert abs(p[0, 0] - want0) < 1e-14
        assert abs(p[0, 1] - (1.0 - want0)) < 1e-14


def test_means_are_over_tokens_not_channels():
    # Block r: tokens alternate a_r + v and a_r - v, so the token mean is a_r
    # exactly, while the channel means differ from token to token.
    r = _rng(3)
    q = r.standard_normal(D)
    A = r.standard_normal((3, D))
    v = 5.0 * r.standard_normal(D)
    K = np.concatenate([np.stack([a + v if t % 2 == 0 else a - v for t in range(B)]) for a in A])
    Q = np.tile(q, (B, 1))
    p = imp.importance(Q, K, B, 1.0)
    z = np.exp(A @ q)
    assert np.allclose(p[0], z / z.sum(), rtol=0, atol=1e-14)


def test_equal_keys_give_uniform_rows():
    r = _rng(4)
    Q = r.standard_normal((2 * B, D))
    k = r.standard_normal(D)
    K = np.tile(k, (7 * B, 1))
    p = imp.importance(Q, K, B, 1.0)
    assert np.all(p == p[:, :1])
    assert np.all(np.abs(p - 1.0 / 7) < 1e-15)


def test_zero_scale_is_uniform():
    r = _rng(5)
    p = imp.importance(r.standard_normal((B, D)), r.standard_normal((5 * B, D)), B, 0.0)
    assert np.all(np.abs(p - 0.2) < 1e-15)


def test_shared_key_shift_and_token_order_invariance():
    r = _rng(6)
    Q = r.standard_normal((2 * B, D))
    K = r.standard_normal((6 * B, D))
    p = imp.importance(Q, K, B, 0.7)
    shifted = imp.importance(Q, K + r.standard_normal(D), B, 0.7)
    assert np.allclose(p, shifted, rtol=1e-12, atol=0)
    perm = np.concatenate([blk * B + r.permutation(B) for blk in range(6)])
    assert np.allclose(p, imp.importance(Q, K[perm], B, 0.7), rtol=1e-12, atol=0)


def test_block_permutation_permutes_columns():
    r = _rng(7)
    Q = r.standard_normal((2 * B, D))
    K = r.standard_normal((5 * B, D))
    sigma = np.array([3, 0, 4, 1, 2])
    Kp = np.concatenate([K[s * B:(s + 1) * B] for s in sigma])
    assert np.allclose(imp.importance(Q, Kp, B, 1.0), imp.importance(Q, K, B, 1.0)[:, sigma],
                       rtol=1e-13, atol=0)


def test_large_scale_concentrates_on_the_best_block():
    r = _rng(8)
    Q = r.standard_normal((B, D))
    K = r.standard_normal((9 * B, D))
    qbar = Q.mean(axis=0)
    best = int(np.argmax(K.reshape(9, B, D).mean(axis=1) @ qbar))
    p = imp.importance(Q, K, B, 1e4)
    assert p[0, best] > 1 - 1e-9


def test_rows_with_far_apart_logits_stay_finite():
    # Each row is normalised on its own: a row whose logits all sit far below
    # another row's must not underflow to 0/0.
    k = np.zeros((3 * B, D))
    k[:B, 0], k[B:2 * B, 0], k[2 * B:, 0] = 1.0, 2.0, 3.0
    Q = np.zeros((2 * B, D))
    Q[:B, 0], Q[B:, 0] = 400.0, -400.0
    p = imp.importance(Q, k, B, 1.0)
    assert np.all(np.isfinite(p))
    assert abs(p[1, 0] - 1.0 / (1.0 + math.exp(-400.0) + math.exp(-800.0))) < 1e-12
