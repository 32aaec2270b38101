"""Pins of routing, probe selection and executed-pair accounting.

Entry masses are pinned by an explicit sort; budget routing by brute force
over every threshold; the tau limits by their closed forms (tau above 1 keeps
every cell, so sparse equals dense; a tiny tau keeps only each group's top
cell); probe apportionment by exact rational arithmetic; rho_exec by the
pages' printed probe density (paperlayer App. A.2).
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import (Params, dense_attention, rho_exec, route_logits, route_masses,
                    route_select, route_to_csr, select_probes, sparsepr_head)


def test_entry_mass_explicit_sort():
    rng = np.random.default_rng(0)
    L = rng.normal(size=(4, 6))
    L[1, 2] = -np.inf
    L[3, :] = 0.0  # all equal: ties go to the lower index
    pi, e, tail, top = route_masses(L)
    for i in range(4):
        fin = [j for j in range(6) if np.isfinite(L[i, j])]
        w = {j: np.exp(L[i, j]) for j in fin}
        z = sum(w.values())
        order = sorted(fin, key=lambda j: (-w[j] / z, j))
        acc = 0.0
        for j in order:
            assert abs(e[i, j] - acc) < 1e-14
            assert abs(pi[i, j] - w[j] / z) < 1e-14
            assert abs(tail[i, j] - sum(w[t] / z for t in order[order.index(j):])) < 1e-14
            assert top[i, j] == (j == order[0])
            acc += w[j] / z
    assert e[1, 2] == np.inf and tail[1, 2] == 0.0
    np.testing.assert_allclose(e[3], np.arange(6) / 6, atol=1e-15)


def test_tau_limits():
    rng = np.random.default_rng(1)
    L = rng.normal(size=(5, 7)) * 3
    cq = np.array([3, 0, 2, 5, 1])
    ck = np.array([2, 2, 0, 4, 1, 3, 1])
    _, e, tail, top = route_masses(route_logits(rng.normal(size=(5, 3)), rng.normal(size=(7, 3)), ck, 1.0))
    allm = route_select(tail, top, cq, ck, "tau", tau=1.5)
    assert (allm == ((cq > 0)[:, None] & (ck > 0)[None, :])).all()
    topm = route_select(tail, top, cq, ck, "tau", tau=1e-12)
    assert topm.sum(1).tolist() == [1, 0, 1, 1, 1]


def test_tail_keeps_peaked_rows_ordered():
    """Entry masses of a very peaked row all round to 1.0; tails stay distinct."""
    L = np.array([[0.0, -40.0, -45.0, -50.0, -60.0]])
    pi, e, tail, top = route_masses(L)
    assert (e[0, 1:] == 1.0).all()
    assert tail[0, 1] > tail[0, 2] > tail[0, 3] > tail[0, 4] > 0
    np.testing.assert_allclose(tail[0, 4], np.exp(-60.0) / np.exp(L[0]).sum(), rtol=1e-12)


def test_budget_brute_force():
    rng = np.random.default_rng(2)
    for trial in range(30):
        Gq, Gk = 4, 5
        cq = rng.integers(0, 6, Gq)
        ck = rng.integers(0, 6, Gk)
        if cq.sum() == 0 or ck.sum() == 0:
            continue
        L = route_logits(rng.normal(size=(Gq, 3)), rng.normal(size=(Gk, 3)) * 2, ck, 1.0)
        _, e, tail, top = route_masses(L)
        rho, M = float(rng.uniform(0.05, 0.9)), int(rng.integers(0, 3))
        got = route_select(tail, top, cq, ck, "budget", rho_target=rho, M=M)
        live = (cq > 0)[:, None] & (ck > 0)[None, :]
        budget = rho * cq.sum() * ck.sum() - M * ck.sum()
        best = None
        for v in sorted(set(tail[live].tolist()), reverse=True):
            keep = live & (tail >= v)
            if (cq[:, None] * ck[None, :])[keep].sum() <= budget:
                best = keep
        want = live & top if best is None else best | (live & top)
        assert (got == want).all()


def test_budget_exact_equality_is_feasible():
    """A threshold whose kept cost equals the budget exactly is taken."""
    cq = np.array([2, 2])
    ck = np.array([2, 2])
    tail = np.array([[1.0, 0.7], [0.4, 1.0]])
    top = np.array([[True, False], [False, True]])
    got = route_select(tail, top, cq, ck, "budget", rho_target=0.75, M=0)  # budget 12 = 3 cells
    assert got.tolist() == [[True, True], [False, True]]
    got = route_select(tail, top, cq, ck, "budget", rho_target=0.75, M=1)  # budget 8: top cells only
    assert got.tolist() == [[True, False], [False, True]]


def test_routing_all_cells_reproduces_dense():
    rng = np.random.default_rng(3)
    N, d = 96, 8
    Q, K, V = rng.normal(size=(N, d)), rng.normal(size=(N, d)), rng.normal(size=(N, d))
    prm = Params(Ms=32, p=4, Gk=6, Gq=5, iters=4, route_mode="tau", tau=2.0, M=0, r=2)
    out = sparsepr_head(Q, K, V, prm)
    np.testing.assert_allclose(out["O"], dense_attention(Q, K, V, 1 / np.sqrt(d)), atol=1e-13)
    assert abs(out["rho_exec"] - 1.0) < 1e-15


def _frac_apportion(counts, M):
    """Largest remainder by exact fractions (independent restatement)."""
    ne = [g for g in range(len(counts)) if counts[g] > 0]
    m = [0] * len(counts)
    for g in ne:
        m[g] = 1
    R, S = M - len(ne), sum(counts) - len(ne)
    if R > 0:
        quota = {g: Fraction(R * (counts[g] - 1), S) for g in ne}
        for g in ne:
            m[g] += int(quota[g])
        left = R - sum(int(q) for q in quota.values())
        order = sorted((g for g in ne if quota[g] != int(quota[g])),
                       key=lambda g: (-(quota[g] - int(quota[g])), g))
        for g in order[:left]:
            m[g] += 1
    return m


def test_probe_apportionment():
    rng = np.random.default_rng(4)
    for trial in range(200):
        G = int(rng.integers(1, 9))
        counts = rng.integers(0, 12, G)
        if counts.sum() == 0:
            continue
        counts[int(rng.integers(0, G))] = max(1, counts[0])
        N = int(counts.sum())
        off = np.concatenate([[0], np.cumsum(counts)])
        perm = rng.permutation(N)
        ne = int((counts > 0).sum())
        M = int(rng.integers(0, N + 1))
        pos, idx, w, m = select_probes(counts, off, perm, M)
        assert m.sum() == M and len(pos) == M
        assert (m <= counts).all()
        if M >= ne:
            assert ((m >= 1) == (counts > 0)).all()
            assert m.tolist() == _frac_apportion(counts.tolist(), M)
        else:
            big = sorted(range(G), key=lambda g: (-counts[g], g))[:M]
            assert sorted(np.nonzero(m)[0].tolist()) == sorted(big)
        assert len(set(pos.tolist())) == M
        for g in range(G):
            pg = [p for p in pos if off[g] <= p < off[g + 1]]
            assert len(pg) == m[g]
            assert pg == [off[g] + ((2 * t + 1) * counts[g]) // (2 * m[g]) for t in range(m[g])]
        if M:
            assert abs(w.sum() - 1.0) < 1e-12 and (idx == perm[pos]).all()


def test_rho_exec_probe_term_matches_pages(golden_dir):
    with open(os.path.join(golden_dir, "probe_density.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    M, lo, hi = int(rows[0][0]), float(rows[0][1]), float(rows[0][2])
    N = int(rows[1][0])
    cq = np.array([N // 2, N - N // 2])
    ck = np.array([N])
    routed, probe, rho = rho_exec(cq, ck, np.array([0, 0, 0]), np.array([], int), M)
    assert routed == 0 and probe == M * N
    assert round(100 * rho, 3) == lo
    # the printed upper end implies the shortest evaluated length, about 44k
    assert 44000 < M / (hi / 100) < 44300
    # a routed cell is counted on top of the probe pairs
    r2 = rho_exec(cq, ck, np.array([0, 1, 1]), np.array([0]), M)
    assert r2[0] == cq[0] * N and r2[2] == pytest.approx((cq[0] * N + M * N) / (N * N))


def test_csr_columns_ascending():
    mask = np.array([[0, 1, 1, 0], [0, 0, 0, 0], [1, 0, 0, 1]], bool)
    rp, ci = route_to_csr(mask)
    assert rp.tolist() == [0, 2, 2, 4] and ci.tolist() == [1, 2, 0, 3]


def _fractions(s):
    return [Fraction(x) for x in s.split(",")]


def test_probe_coverage_weight_values(golden_dir):
    """Probe counts, positions and coverage-weight values on unequal groups,
    worked by hand (tests/golden/probe_coverage_weights.txt): catches an
    inverted or mis-normalised weight that still sums to one."""
    with open(os.path.join(golden_dir, "probe_coverage_weights.txt")) as f:
        cases = [dict(kv.split("=") for kv in line.split()) for line in f
                 if line.strip() and not line.startswith("#")]
    assert len(cases) == 3
    for c in cases:
        counts = np.array([int(x) for x in c["counts"].split(",")], np.int64)
        M = int(c["M"])
        off = np.concatenate([[0], np.cumsum(counts)])
        perm = np.arange(int(counts.sum()))[::-1].copy()  # any permutation
        pos, idx, w, m = select_probes(counts, off, perm, M)
        assert m.tolist() == [int(x) for x in c["m"].split(",")]
        assert pos.tolist() == [int(x) for x in c["pos"].split(",")]
        assert (idx == perm[pos]).all()
        want = [float(x) for x in _fractions(c["w"])]
        np.testing.assert_allclose(w, want, rtol=1e-15, atol=0)
