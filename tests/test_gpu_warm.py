"""GPU warm start: a second call on perturbed inputs (the next denoising step
of the same layer, in miniature) starts its two k-means from the centroids
the first call left in the workspace [paperlayer App. C.1].

The oracle runs its own seeded first call and its own warm second call; the
GPU's warm labels must agree with the oracle's (up to a few rows at a
floating-point near-tie) and its objectives must match; the whole second
call is then checked against the oracle driven by the GPU's labels, as for
every other call.
"""
import numpy as np
import pytest
import torch

import free_block_sparse_means_b200 as spr
from gpu_support import check_head, collect, oracle_params
from oracle import sparsepr_head
from synthetic import voronoi_qkv, workload

pytestmark = pytest.mark.gpu


def _perturbed(t, seed, eps=0.05):
    g = torch.Generator().manual_seed(seed)
    return (t.float() + eps * torch.randn(t.shape, generator=g)).to(torch.bfloat16)


@pytest.mark.parametrize("name,partition", [("tiny", "response"), ("tiny", "semantic"),
                                            ("mid", "response")])
def test_warm_second_call(name, partition):
    wl = workload(name, H=min(workload(name).H, 2), partition=partition)
    Q1, K1, V1 = voronoi_qkv(wl)
    Q2, K2, V2 = (_perturbed(t, 100 + i) for i, t in enumerate((Q1, K1, V1)))
    kw = dict(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, seed=wl.index, route_mode=wl.route_mode,
              tau=wl.tau, rho_target=wl.rho_target, M=wl.M, r=wl.r, lam=wl.lam, partition=partition)
    dev = [t.cuda() for t in (Q1, K1, V1, Q2, K2, V2)]
    O = torch.empty_like(dev[0])
    prm1 = spr.make_params(*dev[:3], O, iters=wl.iters, **kw)
    prm2 = spr.make_params(*dev[3:], O, iters=3, init="warm", **kw)
    ws = spr.alloc_workspace(prm1)
    spr.sparsepr_call(prm1, *dev[:3], O, ws)
    spr.sparsepr_call(prm2, *dev[3:], O, ws)
    stats, err = spr.sparsepr_get_stats(prm2, ws)
    assert err == 0
    g = collect(prm2, ws, Q2, K2, V2, O, stats)
    g["partition"] = partition
    wl2 = wl.replace(iters=3)
    for bh in range(wl.BH):
        b, h = divmod(bh, wl.H)
        args1 = [t[b, h].double().numpy() for t in (Q1, K1, V1)]
        args2 = [t[b, h].double().numpy() for t in (Q2, K2, V2)]
        o1 = sparsepr_head(*args1, oracle_params(wl, partition=partition), bh=bh)
        o2 = sparsepr_head(*args2, oracle_params(wl2, partition=partition), bh=bh,
                           warm=o1["warm_state"])
        agree_k = float((g["lab_k"][bh] == o2["lab_k"]).mean())
        agree_q = float((g["lab_q"][bh] == o2["lab_q"]).mean())
        assert agree_k >= 0.99 and agree_q >= 0.99, (agree_k, agree_q)
        st = g["stats"][bh]
        assert abs(st["obj_k"] - o2["obj_k"]) <= 1e-3 * o2["obj_k"]
        assert abs(st["obj_q"] - o2["obj_q"]) <= 1e-3 * o2["obj_q"]
        check_head(g, wl2, bh)
