"""Pins of Probe-Fitted Residual Reconstruction (paperlayer §4, App. A.3).

A planted affine residual must be recovered exactly on unprobed rows (full
rank with r = d, and low rank with r equal to the planted rank); the subspace
must equal the right singular vectors from numpy's SVD of the weighted
centred residual; the ridge must equal numpy's least squares on the
augmented system; with r = d, lambda -> 0 and every row a probe, the call
returns dense attention.
"""
import numpy as np

from oracle import Params, apply_correction, dense_attention, fit_residual, sparsepr_head


def _planted(M=40, d=6, rank=None, seed=0):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(M + 30, d)) * 2 + 1
    if rank is None:
        B0 = rng.normal(size=(d, d))
        b0 = rng.normal(size=d)
    else:
        A, Bf = rng.normal(size=(d, rank)), rng.normal(size=(rank, d))
        B0 = A @ Bf
        b0 = rng.normal(size=rank) @ Bf  # inside the row space of B0
    D = X + b0 + X @ B0
    w = rng.uniform(0.5, 2.0, M)
    return X, D, w / w.sum(), B0, b0


def test_planted_affine_full_rank_exact():
    X, D, w, B0, b0 = _planted()
    M = len(w)
    U, B, b, sig = fit_residual(X[:M], D[:M], w, r=6, lam=1e-14)
    np.testing.assert_allclose(apply_correction(X[M:], U, B, b), D[M:], atol=1e-8)


def test_planted_affine_low_rank_exact():
    X, D, w, B0, b0 = _planted(d=8, rank=3, seed=1)
    M = len(w)
    U, B, b, sig = fit_residual(X[:M], D[:M], w, r=3, lam=1e-14)
    assert U.shape == (8, 3)
    assert sig[3] < 1e-6 * sig[0]
    np.testing.assert_allclose(apply_correction(X[M:], U, B, b), D[M:], atol=1e-8)
    # asking for more directions than the residual has keeps only 3
    U2, _, _, _ = fit_residual(X[:M], D[:M], w, r=8, lam=1e-14)
    assert U2.shape == (8, 3)


def test_intercept_outside_subspace_kept():
    """Only the feature-dependent term is restricted to U_r: a constant
    residual offset outside the planted row space is still recovered."""
    rng = np.random.default_rng(7)
    X, D, w, B0, b0 = _planted(d=8, rank=2, seed=5)
    M = len(w)
    off = rng.normal(size=8)
    D = D + off
    U, B, b, sig = fit_residual(X[:M], D[:M], w, r=2, lam=1e-14)
    assert U.shape == (8, 2)
    np.testing.assert_allclose(apply_correction(X[M:], U, B, b), D[M:], atol=1e-8)
    # with no usable direction the correction is the weighted mean residual
    U0, B0_, b0_, _ = fit_residual(X[:M], D[:M], w, r=0, lam=1e-3)
    np.testing.assert_allclose(b0_, w @ (D[:M] - X[:M]), atol=1e-12)


def test_subspace_matches_svd_and_ridge_matches_lstsq():
    rng = np.random.default_rng(2)
    M, d, r, lam = 30, 7, 3, 0.05
    X = rng.normal(size=(M, d))
    D = X + rng.normal(size=(M, d)) * np.array([3, 2, 1.5, 0.3, 0.2, 0.1, 0.05])
    w = rng.uniform(0.2, 1.0, M)
    w /= w.sum()
    U, B, b, sig = fit_residual(X, D, w, r, lam)
    R = D - X
    Rc = R - w @ R
    _, sv, Vt = np.linalg.svd(np.sqrt(w)[:, None] * Rc)
    np.testing.assert_allclose(sig, sv, atol=1e-12)
    np.testing.assert_allclose(U @ U.T, Vt[:r].T @ Vt[:r], atol=1e-10)
    # ridge with unpenalised intercept = least squares on the augmented system
    Y = R @ U
    xb, yb = w @ X, w @ Y
    A = np.vstack([np.sqrt(w)[:, None] * (X - xb), np.sqrt(lam) * np.eye(d)])
    rhs = np.vstack([np.sqrt(w)[:, None] * (Y - yb), np.zeros((d, r))])
    Bls = np.linalg.lstsq(A, rhs, rcond=None)[0]
    np.testing.assert_allclose(B, Bls, atol=1e-10)
    np.testing.assert_allclose(b, w @ R - (xb @ Bls) @ U.T, atol=1e-10)


def test_all_rows_probed_returns_dense():
    rng = np.random.default_rng(3)
    N, d = 64, 4
    Q, K, V = rng.normal(size=(N, d)), rng.normal(size=(N, d)), rng.normal(size=(N, d))
    prm = Params(Ms=16, p=3, Gk=4, Gq=4, iters=5, route_mode="tau", tau=0.5, M=N, r=d, lam=1e-12)
    out = sparsepr_head(Q, K, V, prm)
    assert out["rho_exec"] > 1.0  # every probe pair is counted on top of routed cells
    np.testing.assert_allclose(out["O"], dense_attention(Q, K, V, 0.5), atol=1e-13)


def test_zero_residual_gives_no_correction():
    rng = np.random.default_rng(4)
    X = rng.normal(size=(20, 5))
    w = np.full(20, 1 / 20)
    U, B, b, sig = fit_residual(X, X.copy(), w, 3, 1e-3)
    assert U.shape == (5, 0)
    np.testing.assert_allclose(apply_correction(X, U, B, b), X, atol=0)
