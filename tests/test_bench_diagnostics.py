"""The bench's O1 / O2 measurement (torch) agrees with the oracle's
definitions (fp64) on random probability rows with ties."""
import numpy as np
import torch

import bench
from oracle import pooled_support, retained_mass


def test_support_and_mass_match_the_oracle():
    rng = np.random.default_rng(0)
    n, pool, N = 24, 8, 50
    P = rng.dirichlet(np.full(N, 0.3), size=n)
    P[3, :] = 1.0 / N                       # a uniform row: ties everywhere
    P[5, [2, 9]] = P[5, [9, 2]]             # swapped entries
    keep = rng.random((n, N)) < 0.4
    per, pooled, mass = bench.support_and_mass(torch.from_numpy(P), torch.from_numpy(keep), 0.9, pool)
    for b in range(n // pool):
        want_per, want_pooled = pooled_support(P[b * pool:(b + 1) * pool], 0.9)
        np.testing.assert_allclose(per[b * pool:(b + 1) * pool].numpy(), want_per, rtol=0, atol=0)
        assert abs(float(pooled[b]) - want_pooled) == 0.0
    np.testing.assert_allclose(mass.numpy(), retained_mass(P, keep), rtol=1e-12)
