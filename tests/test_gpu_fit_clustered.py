"""The residual fit when the probe residual's spectrum has a tight cluster that
fp32 cannot resolve.

The probe rows' dense outputs are overwritten in the workspace (after the
attention stage) so that the weighted, centred probe residual has a chosen
spectrum: four large directions and a cluster of 40 eigenvalues at about
2e-6 of the largest, spread by far less than an fp32 eigenvalue can be
resolved.  With r = 32 the fit keeps 28 cluster directions, whose individual
eigenvectors are not determined in fp32 while the subspace they span is.
The reconstruction must stay finite and agree with the fp64 oracle's fit
(the cluster carries ~1e-5 of the residual energy, so its basis choice does
not move the output).
"""
import numpy as np
import pytest
import torch

import free_block_sparse_means_b200 as spr
from oracle import apply_correction, fit_residual
from synthetic import voronoi_qkv, workload

pytestmark = pytest.mark.gpu


def test_fit_with_unresolvable_residual_cluster_stays_finite_and_matches():
    wl = workload("mid", H=2, grid=(4, 32, 32), M=256, r=32)
    Q, K, V = (t.cuda() for t in voronoi_qkv(wl))
    O = torch.empty_like(Q)
    prm = spr.make_params(Q, K, V, O, Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, seed=wl.index,
                          route_mode=wl.route_mode, tau=wl.tau, rho_target=wl.rho_target, M=wl.M,
                          r=wl.r, lam=wl.lam)
    ws = spr.alloc_workspace(prm)
    spr.sparsepr_partition(prm, Q, K, V, ws)
    spr.sparsepr_route(prm, ws)
    spr.sparsepr_attend(prm, ws)
    torch.cuda.synchronize()
    BH, N, d, M = wl.BH, wl.N, wl.d, wl.M
    osp = spr.workspace_tensor(prm, ws, "o_sparse", torch.float32, (BH, N, d))
    odn = spr.workspace_tensor(prm, ws, "o_probe", torch.float32, (BH, M, d))
    ppos = spr.workspace_tensor(prm, ws, "probe_pos", torch.int32, (BH, M)).long()
    pw = spr.workspace_tensor(prm, ws, "probe_w", torch.float32, (BH, M))
    perm_q = spr.workspace_tensor(prm, ws, "perm_q", torch.int32, (BH, N)).long().cpu().numpy()
    rng = np.random.default_rng(11)
    spectrum = np.concatenate([[1.0, 0.5, 0.25, 0.125], 2e-6 * (1.0 + 1e-3 * np.arange(40) / 40)])
    sig = np.sqrt(spectrum)
    want_O = []
    for bh in range(BH):
        w = pw[bh].double().cpu().numpy()
        X = osp[bh][ppos[bh]].double().cpu().numpy()
        # Rc = W^-1/2 Qm S V^T with Qm orthonormal and orthogonal to sqrt(w):
        # then sum_t w_t Rc_t = 0 and Rc^T W Rc = V S^2 V^T
        sw = np.sqrt(w)
        A = np.concatenate([sw[:, None], rng.normal(size=(M, len(sig)))], axis=1)
        Qm = np.linalg.qr(A)[0][:, 1:]
        Vb = np.linalg.qr(rng.normal(size=(d, d)))[0][:, :len(sig)]
        R = (Qm * sig[None, :] / sw[:, None]) @ Vb.T * 0.05 + 0.01 * rng.normal(size=d)[None, :]
        D = X + R
        odn[bh] = torch.from_numpy(D).float().cuda()
        # the oracle's fit on the values the GPU sees (fp32-rounded dense rows)
        Df = odn[bh].double().cpu().numpy()
        U, B, b, _ = fit_residual(X, Df, w, wl.r, wl.lam)
        Osp = osp[bh].double().cpu().numpy()
        Oo = apply_correction(Osp, U, B, b)
        Oo[ppos[bh].cpu().numpy()] = Df
        out = np.empty_like(Oo)
        out[perm_q[bh]] = Oo  # back to the original query order
        want_O.append(out)
    torch.cuda.synchronize()
    spr.sparsepr_reconstruct(prm, ws, O)
    stats, err = spr.sparsepr_get_stats(prm, ws)
    assert err == 0
    assert bool(torch.isfinite(O).all())
    got = O.reshape(BH, N, d).double().cpu().numpy()
    for bh in range(BH):
        assert stats[bh]["r_eff"] >= 20, stats[bh]["r_eff"]  # the cluster is inside the rank
        rel = np.linalg.norm(got[bh] - want_O[bh]) / np.linalg.norm(want_O[bh])
        assert rel <= 5e-3, (bh, rel)
