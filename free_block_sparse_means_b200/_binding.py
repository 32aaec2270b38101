"""Thin ctypes binding of libsparsepr.so (the C ABI in include/sparsepr.h).

Argument marshalling only: every step of the SparsePR call runs in the CUDA
library.  PyTorch tensors supply device memory and the CUDA stream.  There is
no CPU fallback: a missing library raises at load time.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libsparsepr.so")

(SPR_OK, SPR_EINVAL, SPR_EUNSUPPORTED, SPR_EWORKSPACE, SPR_ECUDA, SPR_EDEVICE,
 SPR_ESCRATCH) = range(7)
STATUS_NAMES = {0: "SPR_OK", 1: "SPR_EINVAL", 2: "SPR_EUNSUPPORTED", 3: "SPR_EWORKSPACE",
                4: "SPR_ECUDA", 5: "SPR_EDEVICE", 6: "SPR_ESCRATCH"}
ROUTE_TAU, ROUTE_BUDGET = 0, 1
PARTITION_RESPONSE, PARTITION_SEMANTIC = 0, 1
INIT_SEEDED, INIT_WARM = 0, 1
WEIGHTS_COVERAGE, WEIGHTS_UNIFORM = 0, 1
PROBES_STRATIFIED, PROBES_RANKED = 0, 1

VIEWS = {
    "lab_k": 0, "lab_q": 1, "perm_k": 2, "perm_q": 3, "kv_off": 4, "q_off": 5, "row_ptr": 6,
    "col_idx": 7, "probe_pos": 8, "probe_idx": 9, "probe_w": 10, "o_sparse": 11,
    "o_probe": 12, "w_key": 13, "cent_k": 14, "cent_q": 15, "ctilde": 16, "rms": 17,
    "tail": 18, "fit_u": 19, "fit_b": 20, "fit_bvec": 21, "probe_dist": 22,
}


class SprParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
        ("q_strides", ctypes.c_int64 * 3), ("k_strides", ctypes.c_int64 * 3),
        ("v_strides", ctypes.c_int64 * 3), ("o_strides", ctypes.c_int64 * 3),
        ("scale", ctypes.c_float),
        ("Ms", ctypes.c_int32), ("p", ctypes.c_int32), ("Gk", ctypes.c_int32),
        ("Gq", ctypes.c_int32), ("iters", ctypes.c_int32),
        ("seed", ctypes.c_uint64),
        ("route_mode", ctypes.c_int32),
        ("tau", ctypes.c_double), ("rho_target", ctypes.c_double),
        ("M", ctypes.c_int32), ("r", ctypes.c_int32),
        ("lambda_", ctypes.c_double),
        ("partition", ctypes.c_int32), ("init", ctypes.c_int32), ("weights", ctypes.c_int32),
        ("probes", ctypes.c_int32), ("head0", ctypes.c_int32),
    ]


class SprHeadStats(ctypes.Structure):
    _fields_ = [
        ("routed_pairs", ctypes.c_int64), ("probe_pairs", ctypes.c_int64),
        ("nnz_cells", ctypes.c_int64), ("tile_pairs", ctypes.c_int64),
        ("rho_exec", ctypes.c_double), ("obj_k", ctypes.c_double), ("obj_q", ctypes.c_double),
        ("route_threshold", ctypes.c_double),
        ("gk_nonempty", ctypes.c_int32), ("gq_nonempty", ctypes.c_int32),
        ("r_eff", ctypes.c_int32), ("flags", ctypes.c_int32),
    ]


EXPORTS = ["sparsepr_workspace_size", "sparsepr_check_params", "sparsepr_partition",
           "sparsepr_route", "sparsepr_attend", "sparsepr_reconstruct", "sparsepr_call",
           "sparsepr_get_stats", "sparsepr_workspace_view", "sparsepr_version",
           "sparsepr_launch_count", "sparsepr_attend_routed_noalloc"]

_lib = None


def load_library(path: str = LIB_PATH):
    """Load libsparsepr.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libsparsepr.so not built ({path}); run "
                           "`python -m free_block_sparse_means_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(SprParams)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.sparsepr_workspace_size.argtypes = [P]
    lib.sparsepr_workspace_size.restype = sz
    lib.sparsepr_check_params.argtypes = [P]
    lib.sparsepr_check_params.restype = ctypes.c_int
    lib.sparsepr_partition.argtypes = [P, vp, vp, vp, vp, sz, vp]
    lib.sparsepr_partition.restype = ctypes.c_int
    for name in ("sparsepr_route", "sparsepr_attend"):
        getattr(lib, name).argtypes = [P, vp, sz, vp]
        getattr(lib, name).restype = ctypes.c_int
    lib.sparsepr_reconstruct.argtypes = [P, vp, sz, vp, vp]
    lib.sparsepr_reconstruct.restype = ctypes.c_int
    lib.sparsepr_call.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
    lib.sparsepr_call.restype = ctypes.c_int
    lib.sparsepr_get_stats.argtypes = [P, vp, sz, ctypes.POINTER(SprHeadStats),
                                       ctypes.POINTER(ctypes.c_int32), vp]
    lib.sparsepr_get_stats.restype = ctypes.c_int
    lib.sparsepr_workspace_view.argtypes = [P, ctypes.c_int32, ctypes.POINTER(sz),
                                            ctypes.POINTER(sz)]
    lib.sparsepr_workspace_view.restype = ctypes.c_int
    lib.sparsepr_version.argtypes = []
    lib.sparsepr_version.restype = ctypes.c_char_p
    lib.sparsepr_launch_count.argtypes = []
    lib.sparsepr_launch_count.restype = ctypes.c_int64
    i32 = ctypes.c_int32
    lib.sparsepr_attend_routed_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                                   i32, ctypes.c_float, vp, vp, vp]
    lib.sparsepr_attend_routed_noalloc.restype = ctypes.c_int
    _lib = lib
    return lib


class SparsePRError(RuntimeError):
    def __init__(self, where, status):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


def _check(where, status):
    if status != SPR_OK:
        raise SparsePRError(where, status)


def _strides(t: torch.Tensor):
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError("expected a [B, H, N, d] tensor with a contiguous last dimension")
    return (t.stride(0), t.stride(1), t.stride(2))


def make_params(Q, K=None, V=None, O=None, *, Ms, p, Gk, Gq, iters=10, seed=0, route_mode="tau",
                tau=0.9, rho_target=0.25, M=64, r=8, lam=1e-3, scale=0.0,
                partition="response", init="seeded", weights="coverage",
                probes="stratified", head0=0) -> SprParams:
    """spr_params for tensors shaped [B, H, N, d] (strides taken from them)."""
    B, H, N, d = Q.shape
    prm = SprParams()
    prm.B, prm.H, prm.N, prm.d = B, H, N, d
    for name, t in (("q_strides", Q), ("k_strides", K if K is not None else Q),
                    ("v_strides", V if V is not None else Q), ("o_strides", O if O is not None else Q)):
        getattr(prm, name)[:] = _strides(t)
    prm.scale = float(scale)
    prm.Ms, prm.p, prm.Gk, prm.Gq, prm.iters = Ms, p, Gk, Gq, iters
    prm.seed = seed
    prm.route_mode = ROUTE_TAU if route_mode == "tau" else ROUTE_BUDGET
    prm.tau, prm.rho_target = float(tau), float(rho_target)
    prm.M, prm.r, prm.lambda_ = M, r, float(lam)
    if partition not in ("response", "semantic"):
        raise ValueError(f"partition must be 'response' or 'semantic', not {partition!r}")
    prm.partition = PARTITION_RESPONSE if partition == "response" else PARTITION_SEMANTIC
    if init not in ("seeded", "warm"):
        raise ValueError(f"init must be 'seeded' or 'warm', not {init!r}")
    prm.init = INIT_SEEDED if init == "seeded" else INIT_WARM
    if weights not in ("coverage", "uniform"):
        raise ValueError(f"weights must be 'coverage' or 'uniform', not {weights!r}")
    prm.weights = WEIGHTS_COVERAGE if weights == "coverage" else WEIGHTS_UNIFORM
    if probes not in ("stratified", "ranked"):
        raise ValueError(f"probes must be 'stratified' or 'ranked', not {probes!r}")
    prm.probes = PROBES_STRATIFIED if probes == "stratified" else PROBES_RANKED
    prm.head0 = int(head0)
    return prm


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def sparsepr_workspace_size(prm: SprParams) -> int:
    return load_library().sparsepr_workspace_size(ctypes.byref(prm))


def sparsepr_check_params(prm: SprParams) -> int:
    return load_library().sparsepr_check_params(ctypes.byref(prm))


def alloc_workspace(prm: SprParams, device=None) -> torch.Tensor:
    n = sparsepr_workspace_size(prm)
    if n == 0:
        raise SparsePRError("sparsepr_workspace_size", sparsepr_check_params(prm))
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def sparsepr_partition(prm, Q, K, V, ws, stream=None):
    _check("sparsepr_partition", load_library().sparsepr_partition(
        ctypes.byref(prm), Q.data_ptr(), K.data_ptr(), V.data_ptr(), ws.data_ptr(), ws.numel(),
        _stream(stream)))


def sparsepr_route(prm, ws, stream=None):
    _check("sparsepr_route", load_library().sparsepr_route(
        ctypes.byref(prm), ws.data_ptr(), ws.numel(), _stream(stream)))


def sparsepr_attend(prm, ws, stream=None):
    _check("sparsepr_attend", load_library().sparsepr_attend(
        ctypes.byref(prm), ws.data_ptr(), ws.numel(), _stream(stream)))


def sparsepr_reconstruct(prm, ws, O, stream=None):
    _check("sparsepr_reconstruct", load_library().sparsepr_reconstruct(
        ctypes.byref(prm), ws.data_ptr(), ws.numel(), O.data_ptr(), _stream(stream)))


def sparsepr_call(prm, Q, K, V, O, ws, stream=None):
    _check("sparsepr_call", load_library().sparsepr_call(
        ctypes.byref(prm), Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
        ws.data_ptr(), ws.numel(), _stream(stream)))


def sparsepr_get_stats(prm, ws, stream=None, raise_on_device_error=True):
    """Per-head statistics as a list of dicts and the device error word."""
    BH = prm.B * prm.H
    arr = (SprHeadStats * BH)()
    err = ctypes.c_int32(0)
    st = load_library().sparsepr_get_stats(ctypes.byref(prm), ws.data_ptr(), ws.numel(), arr,
                                           ctypes.byref(err), _stream(stream))
    if st != SPR_EDEVICE or raise_on_device_error:
        _check("sparsepr_get_stats", st)
    out = [{f: getattr(s, f) for f, _ in SprHeadStats._fields_} for s in arr]
    return out, err.value


def sparsepr_workspace_view(prm, which) -> tuple:
    off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check("sparsepr_workspace_view", load_library().sparsepr_workspace_view(
        ctypes.byref(prm), VIEWS[which] if isinstance(which, str) else which,
        ctypes.byref(off), ctypes.byref(nb)))
    return off.value, nb.value


def workspace_tensor(prm, ws, which, dtype, shape) -> torch.Tensor:
    """A typed view of one named intermediate buffer inside the workspace."""
    off, nb = sparsepr_workspace_view(prm, which)
    esz = torch.empty((), dtype=dtype).element_size()
    n = 1
    for s in shape:
        n *= s
    if n * esz > nb:
        raise ValueError(f"view {which}: {shape} exceeds {nb} bytes")
    return ws[off:off + n * esz].view(dtype).view(*shape)


def sparsepr_attend_routed_noalloc(Qp, Kp, Vp, q_off, run_ptr, runs, Gk, O, status=None,
                                   scale=0.0, stream=None):
    """Routed attention without device allocation.

    Qp, Kp, Vp: [BH, N, d] bf16 group-major; q_off, run_ptr: [BH, Gq + 1]
    int32; runs: [BH, Gq * Gk, 2] int32 key ranges; O: [BH, N, d] fp32;
    status: optional int32[4] device tensor receiving the device error word.
    Every tensor must be contiguous and on the same CUDA device; anything
    else raises ValueError before the library is called.
    """
    if Qp.dim() != 3:
        raise ValueError("Qp must be [BH, N, d]")
    BH, N, d = Qp.shape
    Gq = q_off.shape[1] - 1 if q_off.dim() == 2 else -1
    want = {"Qp": (Qp, torch.bfloat16, (BH, N, d)), "Kp": (Kp, torch.bfloat16, (BH, N, d)),
            "Vp": (Vp, torch.bfloat16, (BH, N, d)), "q_off": (q_off, torch.int32, (BH, Gq + 1)),
            "run_ptr": (run_ptr, torch.int32, (BH, Gq + 1)),
            "runs": (runs, torch.int32, (BH, Gq * int(Gk), 2)), "O": (O, torch.float32, (BH, N, d))}
    if status is not None:
        want["status"] = (status, torch.int32, (4,))
    for name, (t, dt, shape) in want.items():
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a torch tensor")
        if t.dtype != dt:
            raise ValueError(f"{name} must be {dt}, got {t.dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        if not t.is_cuda or t.device != Qp.device:
            raise ValueError(f"{name} must be on {Qp.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _check("sparsepr_attend_routed_noalloc", load_library().sparsepr_attend_routed_noalloc(
        Qp.data_ptr(), Kp.data_ptr(), Vp.data_ptr(), q_off.data_ptr(), run_ptr.data_ptr(),
        runs.data_ptr(), BH, N, d, Gq, int(Gk), float(scale), O.data_ptr(),
        status.data_ptr() if status is not None else None, _stream(stream)))


def sparsepr_launch_count() -> int:
    """Kernel launches the library has enqueued since it was loaded."""
    return load_library().sparsepr_launch_count()


def sparsepr_version() -> str:
    return load_library().sparsepr_version().decode()
