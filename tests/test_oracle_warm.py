"""Pins of the warm-started k-means (a call starting from the previous call's
centroids [paperlayer App. C.1]).

Continuation: on the same inputs, T1 seeded iterations followed by a warm
call of T2 iterations give the labels of T1 + T2 seeded iterations (both
partitions), which holds only if the previous centroids are mapped into the
new call's coordinates correctly: the raw-key means through W for the keys,
the head-dimension query centroids through Ctilde for the queries.  The warm
state is pinned against the group means of the raw rows.
"""
import dataclasses

import numpy as np
import pytest

from oracle import Params, sparsepr_head


def _inputs(seed, N=160, d=8, centres=5):
    rng = np.random.default_rng(seed)
    mu = 3.0 * rng.normal(size=(centres, d))
    lab = rng.integers(0, centres, size=N)
    return tuple(mu[lab] + rng.normal(size=(N, d)) for _ in range(3))


@pytest.mark.parametrize("partition", ["response", "semantic"])
def test_warm_start_continues_the_seeded_run(partition):
    Q, K, V = _inputs(0)
    base = Params(Ms=64, p=4, Gk=4, Gq=4, iters=3, route_mode="tau", tau=0.9, M=16, r=3,
                  seed=11, partition=partition)
    first = sparsepr_head(Q, K, V, base)
    assert (first["counts_k"] > 0).all() and (first["counts_q"] > 0).all()
    warm = sparsepr_head(Q, K, V, dataclasses.replace(base, iters=4), warm=first["warm_state"])
    cold = sparsepr_head(Q, K, V, dataclasses.replace(base, iters=7))
    assert (warm["lab_k"] == cold["lab_k"]).all()
    assert (warm["lab_q"] == cold["lab_q"]).all()
    assert abs(warm["obj_k"] - cold["obj_k"]) <= 1e-10 * cold["obj_k"]
    assert abs(warm["obj_q"] - cold["obj_q"]) <= 1e-10 * cold["obj_q"]


def test_warm_state_is_raw_group_means():
    Q, K, V = _inputs(1)
    prm = Params(Ms=64, p=4, Gk=4, Gq=4, iters=5, route_mode="tau", tau=0.9, M=16, r=3, seed=2)
    out = sparsepr_head(Q, K, V, prm)
    st = out["warm_state"]
    for g in range(4):
        rows = out["lab_k"] == g
        np.testing.assert_allclose(st["C_raw"][g], K[rows].mean(0), rtol=1e-12, atol=1e-12)
        rq = out["lab_q"] == g
        a = ((out["scale"] / out["rms"][rq])[:, None] * Q[rq]).mean(0)
        np.testing.assert_allclose(st["a_q"][g], a, rtol=1e-12, atol=1e-12)
        # its query-response coordinates are the U-space centroid
        np.testing.assert_allclose(out["Ctilde"] @ st["a_q"][g], out["Cu"][g], rtol=1e-10, atol=1e-12)
