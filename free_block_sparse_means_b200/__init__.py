"""SparsePR sparse attention call for NVIDIA B200 (sm_100a).

The compute lives in ``lib/libsparsepr.so`` (CUDA, built from ``csrc/`` by
``free_block_sparse_means_b200.build``); this package only marshals
arguments to its C ABI.  See ``include/sparsepr.h`` for the contract.
"""
from ._binding import (EXPORTS, LIB_PATH, PARTITION_RESPONSE, PARTITION_SEMANTIC, ROUTE_BUDGET,
                       ROUTE_TAU, VIEWS, SparsePRError, SprHeadStats, SprParams, alloc_workspace,
                       load_library, make_params, sparsepr_attend, sparsepr_attend_routed_noalloc,
                       sparsepr_call, sparsepr_check_params, sparsepr_get_stats,
                       sparsepr_launch_count, sparsepr_partition, sparsepr_reconstruct,
                       sparsepr_route, sparsepr_version, sparsepr_workspace_size,
                       sparsepr_workspace_view, workspace_tensor)
from .host_call import HostPipeline

__all__ = [
    "EXPORTS", "HostPipeline", "LIB_PATH", "PARTITION_RESPONSE", "PARTITION_SEMANTIC", "ROUTE_BUDGET", "ROUTE_TAU",
    "VIEWS", "SparsePRError", "SprHeadStats", "SprParams", "alloc_workspace", "load_library",
    "make_params", "sparsepr_attend", "sparsepr_attend_routed_noalloc", "sparsepr_call",
    "sparsepr_check_params", "sparsepr_get_stats", "sparsepr_launch_count", "sparsepr_partition",
    "sparsepr_reconstruct", "sparsepr_route", "sparsepr_version", "sparsepr_workspace_size",
    "sparsepr_workspace_view", "workspace_tensor",
]
