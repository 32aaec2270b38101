"""Pins of the oracle's whole-call glue on the tiny synthetic workload.

Checked against brute force that does not reuse the step functions: the
sparse output equals a dense softmax masked by the routed (query-group,
K/V-group) cells; rho_exec equals an explicit count of allowed pairs plus
M*N_k; probe rows equal dense rows; the permutations sort the labels;
driven mode with the oracle's own labels reproduces independent mode.
The route logit is pinned by the property that makes it a mass estimate:
when every key of a group equals its centroid, the cell's softmax mass is the
exact attention mass the group's mean query puts on that group.
"""
import numpy as np
import pytest

from oracle import Params, dense_attention, route_logits, route_masses, sparsepr_head
from synthetic import voronoi_qkv, workload


@pytest.fixture(scope="module")
def tiny():
    wl = workload("tiny")
    Q, K, V = voronoi_qkv(wl)
    q, k, v = (t[0, 0].double().numpy() for t in (Q, K, V))
    prm = Params(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters, route_mode="tau",
                 tau=wl.tau, M=wl.M, r=wl.r, lam=wl.lam, seed=wl.index)
    return q, k, v, prm, sparsepr_head(q, k, v, prm, want_dense=True)


def test_sparse_output_is_masked_softmax(tiny):
    q, k, v, prm, out = tiny
    lab_q, lab_k = out["lab_q"], out["lab_k"]
    rp, ci = out["row_ptr"], out["col_idx"]
    allowed = np.zeros((len(q), len(k)), bool)
    for i in range(prm.Gq):
        for j in ci[rp[i]:rp[i + 1]]:
            allowed[np.ix_(lab_q == i, lab_k == j)] = True
    S = out["scale"] * q @ k.T
    S = np.where(allowed, S, -np.inf)
    P = np.exp(S - S.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    np.testing.assert_allclose(out["O_sp"], P @ v, atol=1e-12)
    assert out["routed_pairs"] == allowed.sum()
    assert out["probe_pairs"] == prm.M * len(k)
    assert out["rho_exec"] == pytest.approx((allowed.sum() + prm.M * len(k)) / len(q) ** 2, abs=0)


def test_probe_rows_dense_and_layout(tiny):
    q, k, v, prm, out = tiny
    dense = out["O_dense"]
    np.testing.assert_allclose(out["O"][out["probe_idx"]], dense[out["probe_idx"]], atol=1e-13)
    assert len(set(out["probe_idx"].tolist())) == prm.M
    assert (np.diff(out["lab_q"][out["perm_q"]]) >= 0).all()
    assert (np.diff(out["lab_k"][out["perm_k"]]) >= 0).all()
    assert sorted(out["perm_q"].tolist()) == list(range(len(q)))


def test_route_inputs_and_tau_prefix(tiny):
    """Group means feed the route; each kept set is the mass-ranked prefix."""
    q, k, v, prm, out = tiny
    lab_q, lab_k = out["lab_q"], out["lab_k"]
    for i in range(prm.Gq):
        if (lab_q == i).any():
            np.testing.assert_allclose(out["qbar"][i], q[lab_q == i].sum(0) / (lab_q == i).sum(), atol=1e-13)
    for j in range(prm.Gk):
        if (lab_k == j).any():
            np.testing.assert_allclose(out["C"][j], k[lab_k == j].sum(0) / (lab_k == j).sum(), atol=1e-13)
    rp, ci, pi = out["row_ptr"], out["col_idx"], out["route_pi"]
    for i in range(prm.Gq):
        if not (lab_q == i).any():
            assert rp[i + 1] == rp[i]
            continue
        order = sorted(range(prm.Gk), key=lambda j: (-pi[i, j], j))
        acc, want = 0.0, []
        for j in order:
            if pi[i, j] > 0 and (acc < prm.tau or not want):
                want.append(j)
            acc += pi[i, j]
        assert sorted(want) == ci[rp[i]:rp[i + 1]].tolist()


def test_driven_mode_reproduces_independent(tiny):
    q, k, v, prm, out = tiny
    again = sparsepr_head(q, k, v, prm, lab_k=out["lab_k"], lab_q=out["lab_q"])
    for key in ("perm_q", "q_off", "perm_k", "kv_off", "row_ptr", "col_idx", "probe_idx"):
        assert (again[key] == out[key]).all()
    np.testing.assert_allclose(again["O"], out["O"], atol=0)
    assert again["obj_k"] == pytest.approx(out["kmeans_k_hist"][-1], rel=1e-12)
    assert again["obj_q"] == pytest.approx(out["kmeans_q_hist"][-1], rel=1e-12)


def test_route_logit_is_exact_mass_for_collapsed_groups():
    rng = np.random.default_rng(0)
    d, Gk = 5, 4
    cent = rng.normal(size=(Gk, d))
    sizes = np.array([3, 1, 0, 6])
    keys = np.vstack([np.tile(cent[j], (sizes[j], 1)) for j in range(Gk)])
    lab = np.repeat(np.arange(Gk), sizes)
    qbar = rng.normal(size=(2, d))
    s = 0.8
    pi, _, _, _ = route_masses(route_logits(qbar, cent, sizes, s))
    for i in range(2):
        w = np.exp(s * keys @ qbar[i])
        for j in range(Gk):
            assert abs(pi[i, j] - w[lab == j].sum() / w.sum()) < 1e-13


def test_hunyuan_shape_rows_sample_runs():
    """A sampled-row driven call at reduced length exercises the rows path."""
    wl = workload("sweep", H=1, grid=(2, 16, 32), centers=16, Gk=16, Gq=16, Ms=256, M=64, r=8)
    Q, K, V = voronoi_qkv(wl)
    q, k, v = (t[0, 0].double().numpy() for t in (Q, K, V))
    prm = Params(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters, route_mode="budget",
                 rho_target=0.25, M=wl.M, r=wl.r, lam=wl.lam, seed=wl.index)
    full = sparsepr_head(q, k, v, prm)
    rows = np.array([0, 5, 77, 1023])
    part = sparsepr_head(q, k, v, prm, lab_k=full["lab_k"], lab_q=full["lab_q"], rows=rows)
    np.testing.assert_allclose(part["O"], full["O"][rows], atol=1e-12)
    assert full["rho_exec"] <= 0.25 + 1e-12 or full["row_ptr"][-1] == (full["counts_q"] > 0).sum()
    np.testing.assert_allclose(dense_attention(q[rows], k, v, full["scale"]),
                               sparsepr_head(q, k, v, prm, lab_k=full["lab_k"], lab_q=full["lab_q"],
                                             rows=rows, want_dense=True)["O_dense"], atol=0)


def test_group_means_by_hand_and_empty_groups():
    from oracle import group_means
    X = np.array([[1.0, 2.0], [3.0, 6.0], [10.0, -4.0], [5.0, 5.0]])
    lab = np.array([0, 0, 2, 0])
    got = group_means(X, lab, 4, fallback=np.full((4, 2), 7.0))
    # group 0: rows 0, 1, 3 -> (9/3, 13/3); group 2: row 2; groups 1, 3 keep the fallback
    want = np.array([[3.0, 13.0 / 3.0], [7.0, 7.0], [10.0, -4.0], [7.0, 7.0]])
    assert np.allclose(got, want, rtol=0, atol=1e-15)
    assert np.isnan(group_means(X, lab, 4)[1]).all()  # no fallback: NaN


def test_multi_head_call_slices_per_head_arguments():
    """The [B, H, N, d] wrapper runs head (b, h) as flat head b*H + h: its seeded
    k-means rows and its per-head keyword arrays follow that index."""
    from oracle import sparsepr_call
    wl = workload("tiny", B=2, H=2, grid=(1, 8, 16), centers=8, Gk=8, Gq=8, Ms=64, M=16, r=4)
    Q, K, V = (t.double().numpy() for t in voronoi_qkv(wl))
    prm = Params(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters, route_mode="tau",
                 tau=wl.tau, M=wl.M, r=wl.r, lam=wl.lam, seed=wl.index)
    rows = [np.arange(3 * bh, 3 * bh + 5) for bh in range(4)]
    res = sparsepr_call(Q, K, V, prm, rows=rows)
    for b in range(2):
        for h in range(2):
            bh = 2 * b + h
            one = sparsepr_head(Q[b, h], K[b, h], V[b, h], prm, bh=bh, rows=rows[bh])
            assert np.array_equal(res[bh]["lab_k"], one["lab_k"])
            assert np.array_equal(res[bh]["lab_q"], one["lab_q"])
            assert np.array_equal(res[bh]["O"], one["O"])
