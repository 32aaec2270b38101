"""Pins of the O1 / O2 diagnostics [paperlayer §3.1].

O1 (minimal and pooled support) against brute force over every key subset,
one-hot rows and uniform rows.  O2 (retained mass) through an exact identity
of renormalized hard drop: with retained mass m, o_hd = o_kept and
o_dense - o_hd = (1 - m) (o_drop - o_kept), o_kept and o_drop being the
probability-weighted value means over the kept and dropped keys.
"""
import itertools

import numpy as np

from oracle import (Params, attention_probs, minimal_support, pooled_support, retained_mass,
                    sparsepr_head)


def test_minimal_support_brute_force():
    rng = np.random.default_rng(0)
    for _ in range(20):
        p = rng.dirichlet(np.full(7, 0.6))
        for alpha in (0.5, 0.8, 0.9, 0.99):
            got = minimal_support(p, alpha)
            assert p[got].sum() >= alpha * p.sum() - 1e-15
            best = min(len(c) for n in range(1, 8) for c in itertools.combinations(range(7), n)
                       if p[list(c)].sum() >= alpha * p.sum() - 1e-15)
            assert len(got) == best


def test_support_one_hot_and_uniform_rows():
    N = 16
    P = np.zeros((4, N))
    P[[0, 1, 2, 3], [3, 3, 7, 9]] = 1.0
    per, pooled = pooled_support(P, 0.9)
    assert (per == 1.0 / N).all() and pooled == 3.0 / N
    per, pooled = pooled_support(np.full((3, N), 1.0 / N), 0.5)
    assert (per == 8.0 / N).all() and pooled == 8.0 / N  # ties to the lower index: keys 0..7


def test_retained_mass_identity_of_hard_drop():
    rng = np.random.default_rng(3)
    N, d = 200, 8
    mu = 2.0 * rng.normal(size=(5, d))
    lab = rng.integers(0, 5, size=N)
    Q, K, V = (mu[lab] + rng.normal(size=(N, d)) for _ in range(3))
    prm = Params(Ms=64, p=4, Gk=5, Gq=5, iters=6, route_mode="tau", tau=0.6, M=0, r=0, seed=1)
    out = sparsepr_head(Q, K, V, prm, want_dense=True)
    P = attention_probs(Q, K, out["scale"])
    routed = {i: set(out["col_idx"][out["row_ptr"][i]:out["row_ptr"][i + 1]].tolist())
              for i in range(prm.Gq)}
    keep = np.array([[out["lab_k"][j] in routed[out["lab_q"][i]] for j in range(N)]
                     for i in range(N)])
    m = retained_mass(P, keep)
    assert (m > 0).all() and (m < 1).any()
    o_kept = (P * keep) @ V / m[:, None]
    o_drop = (P * ~keep) @ V / np.maximum(1 - m, 1e-300)[:, None]
    np.testing.assert_allclose(out["O_sp"], o_kept, rtol=1e-10, atol=1e-12)
    err = np.linalg.norm(out["O_dense"] - out["O_sp"], axis=1)
    want = (1 - m) * np.linalg.norm(o_drop - o_kept, axis=1)
    np.testing.assert_allclose(err, want, rtol=1e-8, atol=1e-12)
