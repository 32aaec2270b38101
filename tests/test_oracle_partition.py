"""Pins of the oracle's Response-Coupled Partitioning steps.

Sampling and the metric are pinned by closed forms; key-response coordinates
by the response-profile distance they must reproduce (paperlayer App. B.1:
keys are compared by their pre-softmax responses under the sampled queries);
k-means by brute force over all labelings, monotone objective, exact recovery
and the tie rule; the permutation by a brute-force stable sort; the
query-response coordinates by explicit logits against centred centroids.
"""
import itertools
import os

import numpy as np

from oracle import (group_major_permutation, kmeans, kmeans_init_indices, kmeans_objective,
                    key_response_weights, kv_centroids, query_response_coords,
                    response_metric, sample_query_indices, splitmix64_stream)


def test_sample_indices_closed_form():
    assert sample_query_indices(10, 4).tolist() == [0, 2, 5, 7]
    assert sample_query_indices(7, 7).tolist() == list(range(7))


def test_metric_brute_force():
    rng = np.random.default_rng(0)
    Qs = rng.normal(size=(5, 3))
    MK = response_metric(Qs)
    for a in range(3):
        for b in range(3):
            assert abs(MK[a, b] - sum(Qs[i, a] * Qs[i, b] for i in range(5)) / 5) < 1e-14


def test_key_coords_reproduce_response_profile_distance():
    rng = np.random.default_rng(1)
    d, Ms = 6, 40
    Qs = rng.normal(size=(Ms, d)) @ rng.normal(size=(d, d))
    K = rng.normal(size=(9, d))
    MK = response_metric(Qs)
    W, lam = key_response_weights(MK, d)
    Z = K @ W
    prof = K @ Qs.T  # responses of every key to every sampled query
    for a, b in itertools.combinations(range(9), 2):
        want = ((prof[a] - prof[b]) ** 2).mean() / np.trace(MK)
        assert abs(((Z[a] - Z[b]) ** 2).sum() - want) < 1e-10 * max(1.0, want)


def test_key_coords_diagonal_metric():
    lam = np.array([1.0, 5.0, 3.0, 0.5])
    W, ev = key_response_weights(np.diag(lam), 2)
    np.testing.assert_allclose(ev, [5.0, 3.0, 1.0, 0.5])
    np.testing.assert_allclose(np.abs(W), np.array([[0, 0], [np.sqrt(5 / 9.5), 0],
                                                    [0, np.sqrt(3 / 9.5)], [0, 0]]), atol=1e-14)


def test_splitmix64_published_vectors(golden_dir):
    with open(os.path.join(golden_dir, "splitmix64_vectors.txt")) as f:
        rows = [list(map(int, l.split())) for l in f if l.strip() and not l.startswith("#")]
    for seed, *vals in rows:
        g = splitmix64_stream(seed)
        assert [next(g) for _ in vals] == vals


def test_init_indices_distinct_deterministic():
    a = kmeans_init_indices(100, 30, 7, 3, 0)
    assert len(set(a.tolist())) == 30 and a.min() >= 0 and a.max() < 100
    assert (a == kmeans_init_indices(100, 30, 7, 3, 0)).all()
    assert not (a == kmeans_init_indices(100, 30, 7, 3, 1)).all()
    assert sorted(kmeans_init_indices(12, 12, 1, 0, 0).tolist()) == list(range(12))


def test_init_indices_hand_worked_vectors(golden_dir):
    with open(os.path.join(golden_dir, "kmeans_init_vectors.txt")) as f:
        rows = [list(map(int, l.split())) for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 2
    for n, G, seed, bh, which, *want in rows:
        assert kmeans_init_indices(n, G, seed, bh, which).tolist() == want


def test_kmeans_vs_brute_force_and_monotone():
    rng = np.random.default_rng(2)
    for trial in range(20):
        n, G = int(rng.integers(3, 9)), int(rng.integers(2, 4))
        X = rng.normal(size=(n, 2))
        init = kmeans_init_indices(n, G, trial, 0, 0)
        lab, C, obj, hist = kmeans(X, G, 10, init)
        best = min(kmeans_objective(X, np.array(L), np.array(
            [X[np.array(L) == g].mean(0) if (np.array(L) == g).any() else np.zeros(2) for g in range(G)]))
            for L in itertools.product(range(G), repeat=n))
        assert obj >= best - 1e-12
        assert all(hist[t + 1] <= hist[t] + 1e-12 for t in range(len(hist) - 1))
        # final labels are nearest-centroid of the previous centroids, so a
        # further assignment step cannot lower the objective below obj... and
        # the objective matches the returned centroids
        assert abs(obj - kmeans_objective(X, lab, C)) < 1e-12


def test_kmeans_recovers_separated_clusters_and_ties():
    rng = np.random.default_rng(3)
    centers = np.array([[0, 0], [100, 0], [0, 100]], float)
    truth = rng.integers(0, 3, 60)
    X = centers[truth] + rng.normal(size=(60, 2))
    init = np.array([np.nonzero(truth == g)[0][0] for g in range(3)])
    lab, C, obj, _ = kmeans(X, 3, 5, init)
    assert (lab == truth).all()
    # a point equidistant to two centroids goes to the lower index
    lab2, _, _, _ = kmeans(np.array([[0.0], [2.0], [1.0]]), 2, 1, np.array([0, 1]))
    assert lab2.tolist() == [0, 1, 0]


def test_kmeans_translation_invariant():
    rng = np.random.default_rng(4)
    X = rng.normal(size=(50, 3))
    init = kmeans_init_indices(50, 4, 1, 0, 0)
    a = kmeans(X, 4, 10, init)[0]
    b = kmeans(X + np.array([3.0, -2.0, 7.0]), 4, 10, init)[0]
    assert (a == b).all()


def test_permutation_brute_force():
    rng = np.random.default_rng(5)
    lab = rng.integers(0, 5, 40)
    lab[lab == 3] = 4  # an empty group
    perm, off = group_major_permutation(lab, 6)
    want = sorted(range(40), key=lambda i: (lab[i], i))
    assert perm.tolist() == want
    assert off.tolist() == [0] + list(np.cumsum([np.sum(lab == g) for g in range(6)]))


def test_query_coords_explicit_logits():
    rng = np.random.default_rng(6)
    d, N, Gk = 4, 12, 5
    K, Q = rng.normal(size=(N, d)), rng.normal(size=(7, d))
    lab_k = np.array([0, 0, 1, 1, 1, 3, 3, 4, 4, 4, 0, 1])  # group 2 empty
    C, counts = kv_centroids(K, lab_k, Gk)
    s = 0.5
    U, rms, Ct = query_response_coords(Q, C, counts, s)
    ne = [0, 1, 3, 4]
    cbar = sum(K[lab_k == j].mean(0) for j in ne) / 4
    for i in range(7):
        u = np.array([s * Q[i] @ (K[lab_k == j].mean(0) - cbar) for j in ne])
        r = np.sqrt((u ** 2).mean() + 1e-6)
        np.testing.assert_allclose(U[i], u / r, atol=1e-13)
        assert abs(rms[i] - r) < 1e-13
    # a common shift of every key leaves the coordinates unchanged
    U2, _, _ = query_response_coords(Q, kv_centroids(K + 5.0, lab_k, Gk)[0], counts, s)
    np.testing.assert_allclose(U2, U, atol=1e-12)


def test_kmeans_empty_cluster_keeps_centroid(golden_dir):
    """A cluster that empties at iteration 2 keeps its centroid, which then
    wins a row back at iteration 3 (tests/golden/kmeans_empty_cluster.txt,
    worked by hand): a reset of the empty centroid (to zero, to the data
    mean, or dropped) gives other labels."""
    from fractions import Fraction
    from oracle import kmeans
    rows, init, labels, cents, obj = None, None, {}, {}, {}
    with open(os.path.join(golden_dir, "kmeans_empty_cluster.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            k, *rest = line.split()
            if k == "rows":
                rows = np.array([[float(v) for v in r.split(",")] for r in rest])
            elif k == "init":
                init = [int(v) for v in rest]
            elif k == "labels":
                labels[int(rest[0])] = [int(v) for v in rest[1:]]
            elif k == "centroids":
                cents[int(rest[0])] = [[float(Fraction(v)) for v in r.split(",")] for r in rest[1:]]
            elif k == "objective":
                obj[int(rest[0])] = float(Fraction(rest[1]))
    assert rows is not None and len(labels) == 4
    for T, want in labels.items():
        lab, C, o, hist = kmeans(rows, 3, T, init)
        assert lab.tolist() == want, (T, lab.tolist())
        if T in cents:
            np.testing.assert_allclose(C, cents[T], rtol=0, atol=1e-12)
        if T in obj:
            assert abs(o - obj[T]) < 1e-12
    # the per-iteration objectives are not monotone here only if the rule is
    # wrong: with the kept centroid they never rise
    _, _, _, hist = kmeans(rows, 3, 4, init)
    assert all(b <= a + 1e-12 for a, b in zip(hist, hist[1:]))
