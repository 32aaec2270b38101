"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

Every (batch, head) of the call is independent, so ranks shard heads with no
collective on the data path: each rank takes its own heads (weak scaling) and
the only collectives are the barrier and the max-over-ranks of the timings.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from synthetic import voronoi_qkv, workload


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["RANK"], os.environ["WORLD_SIZE"], os.environ["LOCAL_RANK"] = str(rank), str(world), str(rank)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ws, rk, local = bench.dist_info()
        wl = workload("tiny", H=3)
        heads = bench.shard_heads(wl.BH, rk, ws)
        Q, K, V = voronoi_qkv(wl, heads=heads)
        times = [1.0 + rank, 5.0 - rank, 2.0 * rank]
        mx = bench.reduce_max(times, ws, torch.device("cpu"))
        dist.barrier()
        out[rank] = {"heads": heads, "mx": mx, "q_sum": float(Q.float().sum()),
                     "shape": tuple(Q.shape)}
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_heads_and_reduce_max():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    h0, h1 = res[0]["heads"], res[1]["heads"]
    assert h0 == [0, 1, 2] and h1 == [3, 4, 5]  # disjoint, each rank a full head set
    assert res[0]["mx"] == res[1]["mx"] == [2.0, 5.0, 2.0]
    assert res[0]["shape"] == res[1]["shape"]
    assert res[0]["q_sum"] != res[1]["q_sum"]  # different heads, different data


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max([1.5, 2.5], 1, None) == [1.5, 2.5]
    assert bench.shard_heads(4, 0, 1) == [0, 1, 2, 3]


def test_rank_data_is_reproducible():
    wl = workload("tiny", H=2)
    a = voronoi_qkv(wl, heads=[2, 3])
    b = voronoi_qkv(wl, heads=[2, 3])
    assert all(torch.equal(x, y) for x, y in zip(a, b))
