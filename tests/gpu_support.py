"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
on seeded synthetic inputs, read its intermediates out of the workspace, and
recompute everything downstream of its cluster labels with the oracle
(driven mode), then compare.

Bars (from the method's contract): integer and indexing results bit-exact on
the GPU's labels; k-means objectives within 1e-4 relative; the final output
within 5e-3 per-head relative L2 (bf16 inputs, fp32 accumulation, bf16
output).  The route is evaluated in fp64 on both sides (fp64 group means,
logits, masses and tails), so tail masses agree to 1e-9 relative; a routing
decision that sits on a near-tie (a tail mass within 1e-6 relative of either
side's cut, or two cells of one query group whose masses agree to 1e-9) may
differ.  Such cells are counted, reported and bounded, and the GPU's routed
cells are then handed to the oracle.

The k-means themselves are also compared with the oracle's own, independent
runs from the same seeded initial rows (check_kmeans_independent): label
agreement and objectives, key and query k-means each.
"""
from __future__ import annotations

import numpy as np
import torch

import free_block_sparse_means_b200 as spr
from oracle import Params, sparsepr_head
from synthetic import voronoi_qkv

OUT_TOL = 5e-3
OBJ_TOL = 1e-4
TIE_E = 1e-6
TIE_PI = 1e-9
TAIL_TOL = 1e-9
LABEL_AGREE = 0.99


def oracle_params(wl, **kw) -> Params:
    d = dict(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters, route_mode=wl.route_mode,
             tau=wl.tau, rho_target=wl.rho_target, M=wl.M, r=wl.r, lam=wl.lam, seed=wl.index,
             weights=wl.weights, probe_select=wl.probes)
    d.update(kw)
    return Params(**d)


def run_gpu(wl, N=None, heads=None, inputs=None, check=None, partition=None):
    """Run sparsepr_call on cuda:0; return a dict of CPU numpy results (for
    every head, or only for the head indices in `check`).  The partition
    construction is the workload's unless given."""
    partition = partition or wl.partition
    Q, K, V = inputs if inputs is not None else voronoi_qkv(wl, heads=heads, N=N)
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    Od = torch.empty_like(Qd)
    prm = spr.make_params(Qd, Kd, Vd, Od, Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters,
                          seed=wl.index, route_mode=wl.route_mode, tau=wl.tau,
                          rho_target=wl.rho_target, M=wl.M, r=wl.r, lam=wl.lam,
                          partition=partition, weights=wl.weights, probes=wl.probes)
    ws = spr.alloc_workspace(prm)
    spr.sparsepr_call(prm, Qd, Kd, Vd, Od, ws)
    stats, err = spr.sparsepr_get_stats(prm, ws)
    assert err == 0
    finite = bool(torch.isfinite(Od).all())
    g = collect(prm, ws, Q, K, V, Od, stats, check)
    g["partition"] = partition
    g["all_finite"] = finite
    return g


def collect(prm, ws, Q, K, V, Od, stats, check=None):
    B, H, N, d = prm.B, prm.H, prm.N, prm.d
    BH, Gk, Gq, M = B * H, prm.Gk, prm.Gq, prm.M
    pp = 32  # key coordinates are padded to 32 columns

    sel = list(range(BH)) if check is None else list(check)

    def pick(t):  # a [BH, ...] tensor -> array, or {head: array} for a subset
        if check is None:
            return t.cpu().numpy()
        return {bh: t[bh].cpu().numpy() for bh in sel}

    def view(name, dtype, shape):
        return pick(spr.workspace_tensor(prm, ws, name, dtype, shape))

    i32, f32 = torch.int32, torch.float32
    out = dict(
        prm=prm, stats=stats,
        Q=Q.reshape(BH, N, d), K=K.reshape(BH, N, d), V=V.reshape(BH, N, d),
        O=(Od.float().cpu().reshape(BH, N, d).numpy().astype(np.float64) if check is None else
           {bh: Od.reshape(BH, N, d)[bh].float().cpu().numpy().astype(np.float64) for bh in sel}),
        lab_k=view("lab_k", i32, (BH, N)), lab_q=view("lab_q", i32, (BH, N)),
        perm_k=view("perm_k", i32, (BH, N)), perm_q=view("perm_q", i32, (BH, N)),
        kv_off=view("kv_off", i32, (BH, Gk + 1)), q_off=view("q_off", i32, (BH, Gq + 1)),
        row_ptr=view("row_ptr", i32, (BH, Gq + 1)), col_idx=view("col_idx", i32, (BH, Gq * Gk)),
        tail=view("tail", torch.float64, (BH, Gq, Gk)),
        w_key=view("w_key", f32, (BH, d, pp)), cent_k=view("cent_k", f32, (BH, Gk, pp)),
        o_sparse=view("o_sparse", f32, (BH, N, d)),
    )
    if M > 0:
        out.update(probe_pos=view("probe_pos", i32, (BH, M)), probe_idx=view("probe_idx", i32, (BH, M)),
                   probe_w=view("probe_w", f32, (BH, M)), o_probe=view("o_probe", f32, (BH, M, d)))
        if prm.probes == spr._binding.PROBES_RANKED:
            out["probe_dist"] = view("probe_dist", f32, (BH, N))
    return out


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def gpu_csr(g, bh):
    rp = g["row_ptr"][bh].astype(np.int64)
    return rp, g["col_idx"][bh][: rp[-1]].astype(np.int64)


def mask_from_csr(rp, ci, Gq, Gk):
    m = np.zeros((Gq, Gk), bool)
    for i in range(Gq):
        m[i, ci[rp[i]:rp[i + 1]]] = True
    return m


def fragile_cells(orc, wl, gpu_thr, live):
    """Cells whose routing decision sits on a floating-point near-tie: a tail
    mass within TIE_E (relative) of either side's cut, or a mass that agrees
    with another cell of its row to TIE_PI."""
    tail, pi = orc["route_tail"], orc["route_pi"]
    fr = np.zeros(tail.shape, bool)
    if wl.route_mode == "tau":
        fr |= live & (np.abs(tail - (1.0 - wl.tau)) < TIE_E)
    else:
        keep = orc["_mask"] & live
        thr = tail[keep].min() if keep.any() else 1.0
        for t in (thr, gpu_thr):
            fr |= live & (np.abs(tail - t) <= TIE_E * max(t, 1e-30))
    for i in range(tail.shape[0]):
        row = pi[i]
        srt = np.sort(row[row > 0])
        close = np.nonzero(np.diff(srt) < TIE_PI * max(srt.max() if len(srt) else 1.0, 1e-30))[0]
        for c in close:
            for v in (srt[c], srt[c + 1]):
                fr[i] |= np.isclose(row, v, rtol=0, atol=0)
    return fr


def check_head(g, wl, bh, rows=None, report=None):
    """Driven-mode oracle for one head and every comparison of the contract."""
    prm = oracle_params(wl, partition=g.get("partition", "response"))
    q, k, v = (g[n][bh].double().numpy() for n in ("Q", "K", "V"))
    lab_k, lab_q = g["lab_k"][bh].astype(np.int64), g["lab_q"][bh].astype(np.int64)
    orc = sparsepr_head(q, k, v, prm, bh=bh, lab_k=lab_k, lab_q=lab_q, rows=rows)
    # --- integer / indexing work: bit-exact on the GPU's labels
    assert (g["perm_k"][bh] == orc["perm_k"]).all(), "perm_k"
    assert (g["kv_off"][bh] == orc["kv_off"]).all(), "kv_off"
    assert (g["perm_q"][bh] == orc["perm_q"]).all(), "perm_q"
    assert (g["q_off"][bh] == orc["q_off"]).all(), "q_off"
    rp, ci = gpu_csr(g, bh)
    gm = mask_from_csr(rp, ci, wl.Gq, wl.Gk)
    om = mask_from_csr(orc["row_ptr"], orc["col_idx"], wl.Gq, wl.Gk)
    orc["_mask"] = om
    live = (orc["counts_q"] > 0)[:, None] & (orc["counts_k"] > 0)[None, :]
    # tail masses agree to fp64 accuracy on live cells; dead cells are marked -1.
    # Cells of a row whose masses tie to TIE_PI (relative) may be ranked in
    # either order, which exchanges their tails: such a run of tied cells is
    # compared as a set (sorted tails).
    t_g, t_o = g["tail"][bh].astype(np.float64), orc["route_tail"]
    assert ((t_g < 0) == ~live).all(), "tail liveness"
    pi = orc["route_pi"]
    bad = []
    for i in range(wl.Gq):
        cols = np.nonzero(live[i])[0]
        if len(cols) == 0:
            continue
        cols = cols[np.argsort(-pi[i, cols], kind="stable")]
        start = 0
        for e in range(1, len(cols) + 1):
            if e < len(cols) and pi[i, cols[e - 1]] - pi[i, cols[e]] <= TIE_PI * pi[i, cols[e - 1]]:
                continue
            run = cols[start:e]
            a, b = np.sort(t_g[i, run]), np.sort(t_o[i, run])
            if (np.abs(a - b) > TAIL_TOL * np.maximum(b, 1e-300)).any():
                bad.append((i, [int(c) for c in run], a.tolist(), b.tolist()))
            start = e
    assert not bad, f"tail mass (row, tied run, gpu, oracle): {bad[:4]}"
    near = 0
    if not (gm == om).all():
        fr = fragile_cells(orc, wl, g["stats"][bh]["route_threshold"], live)
        diff = gm != om
        assert not (diff & ~fr).any(), f"route differs off near-ties at {np.argwhere(diff & ~fr)[:5]}"
        near = int(diff.sum())
        orc = sparsepr_head(q, k, v, prm, bh=bh, lab_k=lab_k, lab_q=lab_q, csr=(rp, ci), rows=rows)
    probe_swaps = 0
    if wl.M > 0 and wl.probes == "ranked":
        probe_swaps = check_ranked_probes(g, orc, bh)
        if probe_swaps:
            orc = sparsepr_head(q, k, v, prm, bh=bh, lab_k=lab_k, lab_q=lab_q, csr=gpu_csr(g, bh)
                                if near else None, rows=rows, probe_pos=g["probe_pos"][bh])
    st = g["stats"][bh]
    assert st["routed_pairs"] == orc["routed_pairs"], "routed pairs"
    assert st["probe_pairs"] == orc["probe_pairs"], "probe pairs"
    assert st["nnz_cells"] == len(orc["col_idx"]), "nnz"
    assert st["rho_exec"] == orc["rho_exec"], "rho_exec"
    if wl.M > 0:
        assert (g["probe_pos"][bh] == orc["probe_pos"]).all(), "probe_pos"
        assert (g["probe_idx"][bh] == orc["probe_idx"]).all(), "probe_idx"
        np.testing.assert_allclose(g["probe_w"][bh], orc["probe_w"], rtol=1e-6)
    # --- k-means objectives on the GPU's labels
    ek = abs(st["obj_k"] - orc["obj_k"]) / max(orc["obj_k"], 1e-30)
    eq = abs(st["obj_q"] - orc["obj_q"]) / max(orc["obj_q"], 1e-30)
    # --- floating-point outputs
    want = orc["rows"]
    inv = np.empty_like(g["perm_q"][bh])
    inv[g["perm_q"][bh]] = np.arange(len(inv))
    osp_gpu = g["o_sparse"][bh][inv[want]].astype(np.float64)
    e_sp = rel_l2(osp_gpu, orc["O_sp"])
    e_out = rel_l2(g["O"][bh][want], orc["O"])
    res = dict(bh=bh, near_ties=near, live_cells=int(live.sum()), obj_k_rel=ek, obj_q_rel=eq,
               hard_drop_rel=e_sp, out_rel=e_out, probe_swaps=probe_swaps)
    if wl.M > 0:
        res["probe_rel"] = rel_l2(g["o_probe"][bh].astype(np.float64), orc["probe_dense"])
    if report is not None:
        report.append(res)
    assert ek <= OBJ_TOL, f"key objective rel err {ek}"
    assert eq <= OBJ_TOL, f"query objective rel err {eq}"
    assert e_sp <= OUT_TOL, f"hard-drop output rel-L2 {e_sp}"
    assert e_out <= OUT_TOL, f"output rel-L2 {e_out}"
    if wl.M > 0:
        assert res["probe_rel"] <= OUT_TOL, f"probe rows rel-L2 {res['probe_rel']}"
    return res, orc


DIST_TOL = 2e-5  # ranked probes: fp32 distance error, relative to the group's largest ||u||^2


def check_ranked_probes(g, orc, bh):
    """Distance-ranked probes (reading R16).  The GPU's fp32 distances
    ||u||^2 - 2 (u.c - ||c||^2 / 2) against the oracle's fp64 ||u - c||^2
    (both in permuted order), within DIST_TOL of the group's largest ||u||^2
    (the size the fp32 cancellation error scales with); then, per group,
    the GPU's m_g rows against the oracle's: a row taken by one side only must
    sit within twice that tolerance of the oracle's cut (the m_g-th smallest
    distance).  Returns the number of rows taken differently."""
    perm, qoff = g["perm_q"][bh].astype(np.int64), orc["q_off"]
    d_orc = orc["probe_dist"][perm]
    d_gpu = g["probe_dist"][bh].astype(np.float64)
    u2 = orc["probe_u2"][perm]
    swaps = 0
    gp = g["probe_pos"][bh].astype(np.int64)
    op = orc["probe_pos"].astype(np.int64)
    for gi in range(len(qoff) - 1):
        a, b = int(qoff[gi]), int(qoff[gi + 1])
        if b <= a:
            continue
        scale = float(u2[a:b].max())
        tol = DIST_TOL * max(scale, 1e-30)
        err = np.abs(d_gpu[a:b] - d_orc[a:b])
        assert (err <= tol).all(), f"probe distance group {gi}: max err {err.max()} > {tol}"
        sg = set(gp[(gp >= a) & (gp < b)].tolist())
        so = set(op[(op >= a) & (op < b)].tolist())
        assert len(sg) == len(so), f"probe count group {gi}"
        if sg == so or not so:
            continue
        cut = max(d_orc[p] for p in so)
        for p in sg ^ so:
            assert abs(d_orc[p] - cut) <= 2 * tol, f"probe group {gi}: row at {p} is off the cut"
        swaps += len(sg - so)
    return swaps


def check_kmeans_independent(g, wl, bh, report=None):
    """Each of the GPU's two k-means against the oracle's own, independent run
    of the same k-means (same seeded initial rows, fp64):
      keys:    the oracle's key k-means on the head's inputs;
      queries: the oracle's query k-means on the GPU's key partition (the
               query coordinates are logits against the K/V-group centroids,
               so a few keys on a near-tie that land in another group move
               every query's coordinates; the query k-means is compared on
               the coordinates the GPU's keys define).
    Per k-means: labels equal on at least LABEL_AGREE of the rows and the
    GPU's objective within OBJ_TOL of the oracle's own.  The agreement of the
    GPU's query labels with the fully independent oracle chain is reported."""
    prm = oracle_params(wl, partition=g.get("partition", "response"))
    q, k, v = (g[n][bh].double().numpy() for n in ("Q", "K", "V"))
    none = np.zeros(0, np.int64)
    ind = sparsepr_head(q, k, v, prm, bh=bh, rows=none)
    lab_k = g["lab_k"][bh].astype(np.int64)
    drv = sparsepr_head(q, k, v, prm, bh=bh, lab_k=lab_k, rows=none)
    st = g["stats"][bh]
    agree_k = float((g["lab_k"][bh] == ind["lab_k"]).mean())
    agree_q = float((g["lab_q"][bh] == drv["lab_q"]).mean())
    chain_q = float((g["lab_q"][bh] == ind["lab_q"]).mean())
    ek = abs(st["obj_k"] - ind["obj_k"]) / max(ind["obj_k"], 1e-30)
    eq = abs(st["obj_q"] - drv["obj_q"]) / max(drv["obj_q"], 1e-30)
    res = dict(bh=bh, label_agree_k=agree_k, label_agree_q=agree_q, obj_k_vs_own=ek,
               obj_q_vs_own=eq, label_agree_q_full_chain=chain_q)
    print(f"k-means vs independent oracle: {res}")
    if report is not None:
        report.append(res)
    assert agree_k >= LABEL_AGREE, f"key labels agree {agree_k}"
    assert agree_q >= LABEL_AGREE, f"query labels agree {agree_q}"
    assert ek <= OBJ_TOL, f"key objective vs the oracle's own {ek}"
    assert eq <= OBJ_TOL, f"query objective vs the oracle's own {eq}"
    return res


def near_tie_bound(res, frac=0.005):
    """Near-tie cells stay a small share of the live cells."""
    print(f"route near-ties: head {res['bh']}: {res['near_ties']} of {res['live_cells']} live cells")
    assert res["near_ties"] <= frac * res["live_cells"], res
