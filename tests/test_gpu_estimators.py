"""GPU parity of the estimator variants of the probe-selection / estimator
ablation [paperlayer §5 "Ablations", Table 4]: uniform probe weights (the
unweighted estimator) and r = d (no subspace restriction), against the fp64
oracle driven by the GPU's labels, at the bars of the method's own path.
The r = d cases keep M = 2d probes (with M <= d the ridge system is
underdetermined, the method's conditioning rather than the kernels').
"""
import pytest

from gpu_support import check_head, run_gpu
from synthetic import workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_uniform_weights(name):
    wl = workload(name, H=min(workload(name).H, 2), weights="uniform")
    g = run_gpu(wl)
    for bh in range(wl.BH):
        check_head(g, wl, bh)
        assert abs(float(g["probe_w"][bh].sum()) - 1.0) < 1e-5


@pytest.mark.parametrize("name,r,M", [("tiny", 64, 128), ("mid", 128, 256)])
def test_full_rank_fit(name, r, M):
    wl = workload(name, H=min(workload(name).H, 2), r=r, M=M)
    g = run_gpu(wl)
    for bh in range(wl.BH):
        check_head(g, wl, bh)
        assert g["stats"][bh]["r_eff"] >= 1
