"""The host-buffer call pipelined over chunks of heads (HostPipeline: copies of
one chunk overlap the computation of the next) gives the same output, bit
for bit, as one device call over all heads: heads are independent and each
chunk passes head0, its first flattened head, so the seeded k-means rows are
the same."""
import pytest
import torch

import free_block_sparse_means_b200 as spr
from synthetic import voronoi_qkv, workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("heads_per_chunk", [3, 8])
def test_pipelined_host_call_equals_one_call(heads_per_chunk):
    wl = workload("mid", H=8)
    Q, K, V = voronoi_qkv(wl)
    kw = dict(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters, seed=wl.index,
              route_mode=wl.route_mode, tau=wl.tau, rho_target=wl.rho_target, M=wl.M, r=wl.r,
              lam=wl.lam)
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    Od = torch.empty_like(Qd)
    prm = spr.make_params(Qd, Kd, Vd, Od, **kw)
    ws = spr.alloc_workspace(prm)
    spr.sparsepr_call(prm, Qd, Kd, Vd, Od, ws)
    Qh, Kh, Vh = (t.contiguous().pin_memory() for t in (Q, K, V))
    Oh = torch.empty(Q.shape, dtype=torch.bfloat16).pin_memory()
    pipe = spr.HostPipeline(Q.shape, heads_per_chunk, **kw)
    assert len(pipe.chunks()) == -(-wl.BH // heads_per_chunk)
    for _ in range(2):  # buffers reused across calls
        Oh.zero_()
        pipe(Qh, Kh, Vh, Oh)
        torch.cuda.synchronize()
        assert torch.equal(Oh, Od.cpu())
