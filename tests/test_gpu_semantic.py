"""GPU parity of the semantic-partition comparator (k-means on the raw key and
query rows [paperlayer §2 "Token Partitioning"; §3.1 O3]) against the fp64
oracle on the GPU's own labels: permutations, routing, probes, pair counts
bit-exact; raw-row k-means objectives within 1e-4; outputs within 5e-3
relative L2 (the bars of the response-coupled path).
"""
import pytest

from gpu_support import check_head, run_gpu
from synthetic import workload

pytestmark = pytest.mark.gpu


def test_tiny_semantic_parity():
    wl = workload("tiny")
    g = run_gpu(wl, partition="semantic")
    check_head(g, wl, 0)


def test_mid_semantic_two_heads():
    wl = workload("mid", H=2)
    g = run_gpu(wl, partition="semantic")
    for bh in range(2):
        check_head(g, wl, bh)
        assert 0.2 < g["stats"][bh]["rho_exec"] <= 0.25 + 1e-9


def test_ragged_semantic_more_key_groups():
    # Gk > Gq and a ragged length: the key k-means uses the larger operand rows
    grid = (3, 17, 29)
    n = grid[0] * grid[1] * grid[2]
    wl = workload("mid", H=2, grid=grid, centers=24, Gk=40, Gq=20, Ms=300, p=16, M=256, r=8,
                  route_mode="budget", rho_target=0.3)
    assert n > 256
    g = run_gpu(wl, partition="semantic")
    for bh in range(2):
        check_head(g, wl, bh)
