"""Pins of the oracle's dense attention and renormalized hard drop.

Dense attention is pinned by brute force (explicit sums with math.exp),
closed forms (identical keys give the mean value row; one overwhelming logit
selects its value row) and invariances.  Hard drop is pinned against a masked
dense softmax and against the exact hard-drop residual identity of
paperlayer App. A.1 (the residual depends on the omitted mass and on the
omitted-support output).
"""
import math

import numpy as np

from oracle import attention_rows, dense_attention, hard_drop_attention


def _brute(Q, K, V, s):
    out = []
    for q in Q:
        logits = [s * sum(a * b for a, b in zip(q, k)) for k in K]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = sum(w)
        out.append([sum(w[j] * V[j][c] for j in range(len(K))) / z for c in range(len(V[0]))])
    return np.array(out)


def test_brute_force_tiny():
    rng = np.random.default_rng(0)
    Q, K, V = rng.normal(size=(5, 3)), rng.normal(size=(7, 3)), rng.normal(size=(7, 4))
    np.testing.assert_allclose(attention_rows(Q, K, V, 0.7), _brute(Q, K, V, 0.7), rtol=0, atol=1e-13)


def test_identical_keys_give_mean_value():
    rng = np.random.default_rng(1)
    Q = rng.normal(size=(4, 8))
    K = np.tile(rng.normal(size=(1, 8)), (9, 1))
    V = rng.normal(size=(9, 5))
    np.testing.assert_allclose(attention_rows(Q, K, V, 0.3), np.tile(V.mean(0), (4, 1)), atol=1e-14)


def test_dominant_logit_selects_value_row():
    d = 6
    K = np.eye(d)
    V = np.arange(d * 3, dtype=float).reshape(d, 3)
    Q = 1e3 * np.eye(d)[[2, 4]]
    np.testing.assert_allclose(attention_rows(Q, K, V, 1.0), V[[2, 4]], atol=1e-12)


def test_shift_and_permutation_invariance():
    rng = np.random.default_rng(2)
    Q, K, V = rng.normal(size=(6, 4)), rng.normal(size=(10, 4)), rng.normal(size=(10, 3))
    ref = attention_rows(Q, K, V, 0.5)
    # a constant extra logit per row (extra coordinate q=1, k=c) cancels
    Q2 = np.hstack([Q, np.ones((6, 1))])
    K2 = np.hstack([K, np.full((10, 1), 37.0)])
    np.testing.assert_allclose(attention_rows(Q2, K2, V, 0.5), ref, atol=1e-12)
    perm = rng.permutation(10)
    np.testing.assert_allclose(attention_rows(Q, K[perm], V[perm], 0.5), ref, atol=1e-13)
    np.testing.assert_allclose(dense_attention(Q, K, V, 0.5, chunk=4), ref, atol=0)


def _setup(seed=3, N=24, d=5, Gq=3, Gk=4):
    rng = np.random.default_rng(seed)
    Q, K, V = rng.normal(size=(N, d)), rng.normal(size=(N, d)), rng.normal(size=(N, d))
    lab_q = rng.integers(0, Gq, N)
    lab_k = rng.integers(0, Gk, N)
    return Q, K, V, lab_q, lab_k


def test_hard_drop_equals_masked_softmax():
    Q, K, V, lab_q, lab_k = _setup()
    route = {0: [1, 3], 1: [0], 2: [0, 1, 2, 3]}
    row_ptr = np.array([0, 2, 3, 7])
    col_idx = np.array([1, 3, 0, 0, 1, 2, 3])
    s = 0.4
    got = hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, s)
    # masked dense softmax, written directly
    S = s * Q @ K.T
    allowed = np.array([[lab_k[j] in route[lab_q[i]] for j in range(len(K))] for i in range(len(Q))])
    S = np.where(allowed, S, -np.inf)
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    np.testing.assert_allclose(got, P @ V, atol=1e-13)
    # a subset of rows gives the same rows
    rows = np.array([5, 0, 17])
    np.testing.assert_allclose(hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, s, rows=rows),
                               got[rows], atol=0)


def test_routing_every_cell_is_dense():
    Q, K, V, lab_q, lab_k = _setup(seed=4)
    row_ptr = np.array([0, 4, 8, 12])
    col_idx = np.array([0, 1, 2, 3] * 3)
    np.testing.assert_allclose(hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, 0.4),
                               dense_attention(Q, K, V, 0.4), atol=1e-13)


def test_hard_drop_residual_identity():
    """dense = a*o_ret + (1-a)*o_omit, so R = (1-a)(o_omit - o_ret) (App. A.1)."""
    Q, K, V, lab_q, lab_k = _setup(seed=5)
    row_ptr = np.array([0, 1, 2, 4])
    col_idx = np.array([2, 0, 1, 3])
    s = 0.9
    osp = hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, s)
    dense = dense_attention(Q, K, V, s)
    for i in range(len(Q)):
        cols = col_idx[row_ptr[lab_q[i]]:row_ptr[lab_q[i] + 1]]
        ret = np.isin(lab_k, cols)
        w = np.exp(s * K @ Q[i])
        a = w[ret].sum() / w.sum()
        o_omit = (w[~ret] @ V[~ret]) / w[~ret].sum()
        np.testing.assert_allclose(dense[i] - osp[i], (1 - a) * (o_omit - osp[i]), atol=1e-12)
