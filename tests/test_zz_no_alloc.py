"""The allocation-free routed-attention entry point against the regular
attention stage.

The regular path (partition, route, attend on a workspace) fixes the groups,
the routed cells and the sparse output; the same group-major inputs and
merged key ranges, rebuilt here from the workspace views, go to
sparsepr_attend_routed_noalloc, whose output must equal the stage's bit for
bit (same kernels, same work items).  Several calls in a row share the
library's fixed scratch area, with problems of different sizes in between.
"""
import numpy as np
import pytest
import torch

import free_block_sparse_means_b200 as spr
from synthetic import voronoi_qkv, workload

pytestmark = pytest.mark.gpu


def _regular(wl):
    Q, K, V = (t.cuda() for t in voronoi_qkv(wl))
    prm = spr.make_params(Q, Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, seed=wl.index,
                          route_mode=wl.route_mode, tau=wl.tau, rho_target=wl.rho_target, M=wl.M,
                          r=wl.r, lam=wl.lam)
    ws = spr.alloc_workspace(prm)
    spr.sparsepr_partition(prm, Q, K, V, ws)
    spr.sparsepr_route(prm, ws)
    spr.sparsepr_attend(prm, ws)
    torch.cuda.synchronize()
    BH, N, d, Gq, Gk = wl.BH, wl.N, wl.d, wl.Gq, wl.Gk

    def view(name, dtype, shape):
        return spr.workspace_tensor(prm, ws, name, dtype, shape).clone()

    perm_q = view("perm_q", torch.int32, (BH, N)).long()
    perm_k = view("perm_k", torch.int32, (BH, N)).long()
    q_off = view("q_off", torch.int32, (BH, Gq + 1))
    kv_off = view("kv_off", torch.int32, (BH, Gk + 1)).cpu().numpy()
    row_ptr = view("row_ptr", torch.int32, (BH, Gq + 1)).cpu().numpy()
    col_idx = view("col_idx", torch.int32, (BH, Gq * Gk)).cpu().numpy()
    o_sparse = view("o_sparse", torch.float32, (BH, N, d))

    def group_major(t, perm):
        t = t.reshape(BH, N, d)
        return torch.gather(t, 1, perm[:, :, None].expand(BH, N, d)).contiguous()

    # Merged key ranges: consecutive routed K/V groups whose keys are
    # adjacent in the permuted order form one range.
    run_ptr = np.zeros((BH, Gq + 1), np.int32)
    runs = np.zeros((BH, Gq * Gk, 2), np.int32)
    for bh in range(BH):
        nr = 0
        for i in range(Gq):
            run_ptr[bh, i] = nr
            end = -1
            for j in col_idx[bh, row_ptr[bh, i]:row_ptr[bh, i + 1]]:
                a, b = kv_off[bh, j], kv_off[bh, j + 1]
                if a != end:
                    runs[bh, nr] = (a, b)
                    nr += 1
                else:
                    runs[bh, nr - 1, 1] = b
                end = b
        run_ptr[bh, Gq] = nr
    return dict(Qp=group_major(Q, perm_q), Kp=group_major(K, perm_k), Vp=group_major(V, perm_k),
                q_off=q_off, run_ptr=torch.from_numpy(run_ptr).cuda(),
                runs=torch.from_numpy(runs).cuda(), Gk=Gk, o_sparse=o_sparse, wl=wl)


def _noalloc(c, status, O=None):
    if O is None:
        O = torch.empty_like(c["o_sparse"])
    O.fill_(float("nan"))
    spr.sparsepr_attend_routed_noalloc(c["Qp"], c["Kp"], c["Vp"], c["q_off"], c["run_ptr"],
                                       c["runs"], c["Gk"], O, status=status)
    return O


def _rows_against_definition(c, O, rows_per_head=6, seed=0):
    """A few rows of each head against softmax over the union of their ranges (fp64)."""
    g = np.random.default_rng(seed)
    q_off = c["q_off"].cpu().numpy()
    run_ptr, runs = c["run_ptr"].cpu().numpy(), c["runs"].cpu().numpy()
    BH, N, d = O.shape
    scale = 1.0 / np.sqrt(d)
    for bh in range(BH):
        q = c["Qp"][bh].double().cpu().numpy()
        k = c["Kp"][bh].double().cpu().numpy()
        v = c["Vp"][bh].double().cpu().numpy()
        for r in g.integers(0, N, rows_per_head):
            i = int(np.searchsorted(q_off[bh], r, side="right") - 1)
            keys = np.concatenate([np.arange(x, y) for x, y in
                                   runs[bh, run_ptr[bh, i]:run_ptr[bh, i + 1]]])
            s = scale * (k[keys] @ q[r])
            w = np.exp(s - s.max())
            want = (w / w.sum()) @ v[keys]
            got = O[bh, r].double().cpu().numpy()
            assert np.linalg.norm(got - want) <= 5e-3 * np.linalg.norm(want), (bh, r)


def test_noalloc_equals_attend_stage_over_consecutive_calls():
    a = _regular(workload("mid", H=2, grid=(2, 32, 32)))  # d = 128, 2048 tokens
    b = _regular(workload("tiny"))  # d = 64, 1024 tokens
    status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    outs = {id(a): torch.empty_like(a["o_sparse"]), id(b): torch.empty_like(b["o_sparse"])}
    free = []
    for c in (a, b, a, b):
        O = _noalloc(c, status, outs[id(c)])
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        assert status.tolist() == [0, 0, 0, 0]
        assert torch.equal(O, c["o_sparse"])
    # after the first call on the device, calls take no device memory
    assert free[1] == free[2] == free[3]
    _rows_against_definition(a, outs[id(a)])
    _rows_against_definition(b, outs[id(b)])


def test_noalloc_bad_range_reports_and_next_call_recovers():
    c = _regular(workload("tiny"))
    bad = c["runs"].clone()
    bad[0, 0, 1] = c["wl"].N + 5  # a key range past the end of the head
    status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    O = torch.full_like(c["o_sparse"], float("nan"))
    spr.sparsepr_attend_routed_noalloc(c["Qp"], c["Kp"], c["Vp"], c["q_off"], c["run_ptr"], bad,
                                       c["Gk"], O, status=status)
    torch.cuda.synchronize()
    st = status.tolist()
    assert st[0] == 1 and st[1] == 0 and st[3] == 2, st
    assert torch.isnan(O).all()  # nothing computed
    O2 = _noalloc(c, status)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0, 0, 0]
    assert torch.equal(O2, c["o_sparse"])
