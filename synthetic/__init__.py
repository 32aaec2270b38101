"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This package draws inputs only; it holds none of the sparse-attention method's
arithmetic.
"""
from .voronoi import WORKLOADS, Workload, voronoi_head, voronoi_qkv, workload

__all__ = ["WORKLOADS", "Workload", "voronoi_head", "voronoi_qkv", "workload"]
