"""Pins of the distance-ranked probe selection (a probe-selection variant of
the pages' ablation): per-group counts and weights equal to the stratified
selection; within a group the chosen rows are the nearest to the centroid
(brute force over every subset on small groups), ties to the lower original
index (equal distances give the first rows).
"""
import dataclasses
import itertools

import numpy as np

from oracle import Params, select_probes, sparsepr_head


def _groups(seed, G=4, n=40):
    rng = np.random.default_rng(seed)
    lab = rng.integers(0, G, size=n)
    perm = np.argsort(lab, kind="stable")
    counts = np.bincount(lab, minlength=G)
    off = np.concatenate([[0], np.cumsum(counts)])
    return lab, perm, counts, off


def test_counts_and_weights_match_stratified():
    lab, perm, counts, off = _groups(0)
    dist = np.random.default_rng(1).random(len(lab))
    a = select_probes(counts, off, perm, 13)
    b = select_probes(counts, off, perm, 13, dist)
    assert (a[3] == b[3]).all()
    np.testing.assert_array_equal(a[2], b[2])


def test_nearest_rows_by_brute_force():
    lab, perm, counts, off = _groups(2, G=3, n=18)
    dist = np.random.default_rng(3).random(len(lab))
    pos, idx, _, m = select_probes(counts, off, perm, 7, dist)
    for g in range(3):
        members = perm[off[g]:off[g + 1]]
        got = sorted(idx[(pos >= off[g]) & (pos < off[g + 1])].tolist())
        best = min(itertools.combinations(members.tolist(), int(m[g])),
                   key=lambda c: sum(dist[list(c)]))
        assert got == sorted(best)


def test_equal_distances_take_the_first_rows():
    lab, perm, counts, off = _groups(4)
    pos, idx, _, m = select_probes(counts, off, perm, 9, np.zeros(len(lab)))
    for g in range(len(counts)):
        members = perm[off[g]:off[g + 1]]
        got = idx[(pos >= off[g]) & (pos < off[g + 1])]
        assert got.tolist() == sorted(members.tolist())[: int(m[g])]


def test_ranked_call_keeps_the_nearest_rows():
    rng = np.random.default_rng(5)
    N, d = 160, 8
    mu = 2.0 * rng.normal(size=(4, d))
    lab = rng.integers(0, 4, size=N)
    Q, K, V = (mu[lab] + rng.normal(size=(N, d)) for _ in range(3))
    for partition in ("response", "semantic"):
        prm = Params(Ms=64, p=4, Gk=4, Gq=4, iters=6, route_mode="tau", tau=0.8, M=16, r=3,
                     seed=3, partition=partition, probe_select="ranked")
        out = sparsepr_head(Q, K, V, prm)
        dist, lq = out["probe_dist"], out["lab_q"]
        chosen = np.zeros(N, bool)
        chosen[out["probe_idx"]] = True
        for g in range(4):
            inside = lq == g
            if chosen[inside].any() and (~chosen[inside]).any():
                assert dist[inside & chosen].max() <= dist[inside & ~chosen].min()
        strat = sparsepr_head(Q, K, V, dataclasses.replace(prm, probe_select="stratified"))
        assert (np.bincount(lq[out["probe_idx"]], minlength=4) ==
                np.bincount(strat["lab_q"][strat["probe_idx"]], minlength=4)).all()
