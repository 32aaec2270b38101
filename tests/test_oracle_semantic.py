"""Pins of the semantic-partition comparator and of the O3 diagnostic.

The semantic partition [paperlayer §2 "Token Partitioning"; §3.1 O3] clusters
the raw key and the raw query rows independently.  Pinned by: its key groups
do not depend on the queries (nor its query groups on the keys), unlike the
response-coupled groups; on two well-separated planted clusters it reaches
the brute-force optimum over every labeling; its objectives are the raw-row
ones.  The O3 decomposition [paperlayer §3.1 O3] is pinned by a residual that
is exactly affine in the sparse output, one orthogonal to every affine
feature, Pythagoras on random data, invariance to an invertible affine change
of the features, and a one-feature closed form (simple regression).
"""
import itertools

import numpy as np

from oracle import Params, affine_residual_decomposition, kmeans_objective, sparsepr_head


def _inputs(seed, N=96, d=8):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(N, d)), rng.normal(size=(N, d)), rng.normal(size=(N, d)))


def _params(partition, **kw):
    base = dict(Ms=32, p=4, Gk=4, Gq=4, iters=8, route_mode="tau", tau=0.9, M=12, r=3, lam=1e-3,
                seed=5, partition=partition)
    base.update(kw)
    return Params(**base)


def test_semantic_key_groups_ignore_queries_and_vice_versa():
    Q, K, V = _inputs(0)
    Q2 = Q + np.random.default_rng(9).normal(size=Q.shape)
    K2 = K + np.random.default_rng(8).normal(size=K.shape)
    a = sparsepr_head(Q, K, V, _params("semantic"))
    b = sparsepr_head(Q2, K, V, _params("semantic"))
    c = sparsepr_head(Q, K2, V, _params("semantic"))
    assert (a["lab_k"] == b["lab_k"]).all()
    assert (a["lab_q"] == c["lab_q"]).all()
    # the response-coupled key groups do depend on the queries
    r1 = sparsepr_head(Q, K, V, _params("response"))
    r2 = sparsepr_head(Q2, K, V, _params("response"))
    assert (r1["lab_k"] != r2["lab_k"]).any() or (r1["Z"] != r2["Z"]).any()


def test_semantic_reaches_brute_force_optimum_on_separated_clusters():
    rng = np.random.default_rng(3)
    d, N = 3, 10
    centres = np.array([[10.0, 0, 0], [-10.0, 0, 0]])
    truth = np.array([0, 1] * (N // 2))
    X = centres[truth] + 0.1 * rng.normal(size=(N, d))
    out = sparsepr_head(X, X, X, _params("semantic", Gk=2, Gq=2, iters=20, M=0))
    best = min(kmeans_objective(X, np.array(lab), np.array([X[np.array(lab) == g].mean(0) if
                                                            (np.array(lab) == g).any() else
                                                            np.zeros(d) for g in range(2)]))
               for lab in itertools.product(range(2), repeat=N) if len(set(lab)) == 2)
    assert abs(out["obj_k"] - best) <= 1e-9 * best
    assert abs(out["obj_q"] - best) <= 1e-9 * best
    # the planted split, up to the names of the groups
    assert len(set(zip(out["lab_k"].tolist(), truth.tolist()))) == 2


def test_semantic_objectives_are_raw_row_sums():
    Q, K, V = _inputs(1)
    out = sparsepr_head(Q, K, V, _params("semantic"))
    for X, lab, key in ((K, out["lab_k"], "obj_k"), (Q, out["lab_q"], "obj_q")):
        tot = 0.0
        for g in np.unique(lab):
            rows = X[lab == g]
            tot += ((rows - rows.mean(0)) ** 2).sum()
        assert abs(out[key] - tot) <= 1e-10 * tot


def test_o3_exactly_affine_residual():
    rng = np.random.default_rng(4)
    X = rng.normal(size=(50, 6))
    R = X @ rng.normal(size=(6, 6)) + rng.normal(size=(1, 6))
    dec = affine_residual_decomposition(X, X + R)
    assert abs(dec["affine_fraction"] - 1.0) < 1e-12
    assert dec["orthogonal_energy"] <= 1e-20 * dec["residual_energy"]


def test_o3_residual_orthogonal_to_features():
    rng = np.random.default_rng(5)
    X = rng.normal(size=(40, 4))
    F = np.concatenate([X, np.ones((40, 1))], axis=1)
    Rr = rng.normal(size=(40, 4))
    R = Rr - F @ np.linalg.solve(F.T @ F, F.T @ Rr)  # remove the feature span by normal equations
    dec = affine_residual_decomposition(X, X + R)
    assert dec["affine_fraction"] < 1e-20
    assert abs(dec["orthogonal_energy"] - (R * R).sum()) <= 1e-12 * (R * R).sum()


def test_o3_pythagoras_and_affine_invariance():
    rng = np.random.default_rng(6)
    X = rng.normal(size=(60, 5))
    Od = rng.normal(size=(60, 5))
    dec = affine_residual_decomposition(X, Od)
    assert abs(dec["affine_energy"] + dec["orthogonal_energy"] - dec["residual_energy"]) <= \
        1e-12 * dec["residual_energy"]
    # the same residual with features X A + c (A invertible): same split
    A, c = rng.normal(size=(5, 5)), rng.normal(size=(1, 5))
    Xp = X @ A + c
    dec2 = affine_residual_decomposition(Xp, Xp + (Od - X))
    for k in ("affine_energy", "orthogonal_energy", "residual_energy"):
        assert abs(dec2[k] - dec[k]) <= 1e-9 * dec["residual_energy"]


def test_o3_one_feature_closed_form():
    rng = np.random.default_rng(7)
    x = rng.normal(size=30)
    r = 0.7 * x + rng.normal(size=30)
    dec = affine_residual_decomposition(x[:, None], (x + r)[:, None])
    xc, rc = x - x.mean(), r - r.mean()
    slope = (xc * rc).sum() / (xc * xc).sum()
    fit = r.mean() + slope * xc
    assert abs(dec["affine_energy"] - (fit * fit).sum()) <= 1e-12 * (r * r).sum()
    assert abs(dec["orthogonal_energy"] - ((r - fit) ** 2).sum()) <= 1e-12 * (r * r).sum()
