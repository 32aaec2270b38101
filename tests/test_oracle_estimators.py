"""Pins of the estimator variants of the probe-selection / estimator ablation
[paperlayer §5 "Ablations", Table 4]: the unweighted estimator (every probe
weighs 1/M) and the estimator without the subspace restriction (r = d).

r = d is pinned against the full weighted ridge estimator written out
directly (normal equations, no eigendecomposition): correction(x) = Rbar +
(x - xbar) B with B = (Xc^T W Xc + lambda I)^-1 Xc^T W Rc.  Uniform weights
are pinned by their values and by coinciding with coverage weights when every
probed group has the same size and the same probe count.
"""
import dataclasses

import numpy as np

from oracle import Params, sparsepr_head


def _inputs(seed, N=256, d=8, centres=6):
    rng = np.random.default_rng(seed)
    mu = 2.0 * rng.normal(size=(centres, d))
    lab = rng.integers(0, centres, size=N)
    return tuple(mu[lab] + rng.normal(size=(N, d)) for _ in range(3))


BASE = Params(Ms=64, p=4, Gk=6, Gq=6, iters=6, route_mode="tau", tau=0.5, M=48, r=3, lam=1e-2,
              seed=4)


def test_uniform_weights_values():
    Q, K, V = _inputs(0)
    out = sparsepr_head(Q, K, V, dataclasses.replace(BASE, weights="uniform"))
    w = out["probe_w"]
    assert len(w) == BASE.M and np.all(w == 1.0 / BASE.M)


def test_uniform_equals_coverage_when_groups_balanced():
    Q, K, V = _inputs(1, N=240)
    lab_q = np.repeat(np.arange(6), 40)  # six groups of 40, M = 48: eight probes each
    a = sparsepr_head(Q, K, V, BASE, lab_q=lab_q)
    b = sparsepr_head(Q, K, V, dataclasses.replace(BASE, weights="uniform"), lab_q=lab_q)
    np.testing.assert_allclose(a["probe_w"], b["probe_w"], rtol=1e-15)
    np.testing.assert_allclose(a["O"], b["O"], rtol=1e-12, atol=1e-14)


def test_full_rank_fit_is_the_unrestricted_ridge_estimator():
    Q, K, V = _inputs(2)
    d = Q.shape[1]
    for weights in ("coverage", "uniform"):
        prm = dataclasses.replace(BASE, r=d, weights=weights)
        out = sparsepr_head(Q, K, V, prm)
        X, D, w = out["probe_sparse"], out["probe_dense"], out["probe_w"]
        R = D - X
        xbar, rbar = w @ X, w @ R
        Xc, Rc = X - xbar, R - rbar
        B = np.linalg.solve(Xc.T @ (w[:, None] * Xc) + prm.lam * np.eye(d), Xc.T @ (w[:, None] * Rc))
        want = out["O_sp"] + rbar + (out["O_sp"] - xbar) @ B
        probe = np.isin(out["rows"], out["probe_idx"])
        np.testing.assert_allclose(out["O"][~probe], want[~probe], rtol=1e-9, atol=1e-12)
