"""CPU checks of the C-ABI library: it loads, exports every function that
include/sparsepr.h declares, the ctypes structs match the C layout (checked by
compiling a probe against the header with gcc), and argument validation
rejects bad parameters without touching a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import free_block_sparse_means_b200 as spr
from free_block_sparse_means_b200 import build as spr_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparsepr.h")


@pytest.fixture(scope="module")
def lib():
    spr_build.build()
    return spr.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sparsepr_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(spr.EXPORTS) == names
    out = subprocess.run(["nm", "-D", "--defined-only", spr.LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_struct_layout_matches_c(tmp_path):
    probe = tmp_path / "probe.c"
    probe.write_text('''
#include <stdio.h>
#include <stddef.h>
#include "sparsepr.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\\n", sizeof(spr_params),
         offsetof(spr_params, scale), offsetof(spr_params, seed), offsetof(spr_params, tau),
         offsetof(spr_params, M), offsetof(spr_params, lambda), offsetof(spr_params, partition),
         offsetof(spr_params, init), offsetof(spr_params, weights), offsetof(spr_params, probes),
         offsetof(spr_params, head0), sizeof(spr_head_stats),
         offsetof(spr_head_stats, gk_nonempty));
  return 0;
}
''')
    exe = tmp_path / "probe"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(probe), "-o", str(exe)])
    got = list(map(int, subprocess.check_output([str(exe)]).split()))
    P, S = spr.SprParams, spr.SprHeadStats
    want = [ctypes.sizeof(P), P.scale.offset, P.seed.offset, P.tau.offset, P.M.offset,
            P.lambda_.offset, P.partition.offset, P.init.offset, P.weights.offset,
            P.probes.offset, P.head0.offset, ctypes.sizeof(S), S.gk_nonempty.offset]
    assert got == want


def _params(**kw):
    Q = torch.empty(1, 2, 4096, 128, dtype=torch.bfloat16)
    base = dict(Ms=256, p=32, Gk=64, Gq=64, M=128, r=16, route_mode="budget", rho_target=0.25)
    base.update(kw)
    return spr.make_params(Q, **base)


def test_validation(lib):
    assert spr.sparsepr_check_params(_params()) == 0
    bad = [dict(Ms=0), dict(Ms=5000), dict(p=0), dict(p=65), dict(Gk=0), dict(Gq=300),
           dict(iters=0), dict(M=-1), dict(M=5000), dict(r=129), dict(lam=-1.0),
           dict(route_mode="tau", tau=0.0), dict(rho_target=0.0)]
    for kw in bad:
        assert spr.sparsepr_check_params(_params(**kw)) in (1, 2), kw
        assert spr.sparsepr_workspace_size(_params(**kw)) == 0, kw
    prm = _params()
    prm.d = 96
    assert spr.sparsepr_check_params(prm) == spr._binding.SPR_EUNSUPPORTED
    # key coordinates are padded to 32 columns: p up to 32
    assert spr.sparsepr_check_params(_params(p=33)) == spr._binding.SPR_EUNSUPPORTED
    assert spr.sparsepr_check_params(_params(p=7)) == 0
    assert spr.sparsepr_check_params(_params(partition="semantic")) == 0
    # distance-ranked probes need the query-response coordinates
    assert spr.sparsepr_check_params(_params(probes="ranked")) == 0
    assert spr.sparsepr_check_params(_params(probes="ranked", partition="semantic")) == \
        spr._binding.SPR_EUNSUPPORTED
    assert spr.sparsepr_check_params(_params(head0=23)) == 0
    assert spr.sparsepr_check_params(_params(head0=-1)) == spr._binding.SPR_EINVAL
    for field in ("partition", "init", "weights", "probes"):
        prm = _params()
        setattr(prm, field, 2)
        assert spr.sparsepr_check_params(prm) == spr._binding.SPR_EINVAL, field
        assert spr.sparsepr_workspace_size(prm) == 0, field
    assert spr.sparsepr_check_params(_params(init="warm", weights="uniform")) == 0
    # the options do not change the workspace a call needs
    n = spr.sparsepr_workspace_size(_params())
    assert spr.sparsepr_workspace_size(_params(init="warm", weights="uniform", partition="semantic")) == n
    assert spr.sparsepr_workspace_size(_params(probes="ranked")) == n


def test_entry_points_reject_before_any_gpu_work(lib):
    prm = _params()
    n = spr.sparsepr_workspace_size(prm)
    assert n > 0
    # null workspace, short workspace, misaligned workspace: rejected on the host
    assert lib.sparsepr_route(ctypes.byref(prm), None, n, None) == spr._binding.SPR_EWORKSPACE
    assert lib.sparsepr_attend(ctypes.byref(prm), 256, n - 1, None) == spr._binding.SPR_EWORKSPACE
    assert lib.sparsepr_attend(ctypes.byref(prm), 257, n, None) == spr._binding.SPR_EWORKSPACE
    assert lib.sparsepr_call(ctypes.byref(prm), 256, 256, 256, None, 256, n, None) == \
        spr._binding.SPR_EINVAL
    # misaligned token stride
    prm2 = _params()
    prm2.q_strides[2] = 100
    assert lib.sparsepr_partition(ctypes.byref(prm2), 256, 256, 256, 256, n, None) == \
        spr._binding.SPR_EUNSUPPORTED
    bad = _params(Gk=0)
    assert lib.sparsepr_call(ctypes.byref(bad), 256, 256, 256, 256, 256, n, None) == \
        spr._binding.SPR_EINVAL


def test_workspace_views_in_bounds(lib):
    prm = _params()
    n = spr.sparsepr_workspace_size(prm)
    for name in spr.VIEWS:
        off, nb = spr.sparsepr_workspace_view(prm, name)
        assert off % 256 == 0 and nb > 0 and off + nb <= n, name
    with pytest.raises(spr.SparsePRError):
        spr.sparsepr_workspace_view(prm, 99)


def test_workspace_scales_with_problem(lib):
    small = spr.sparsepr_workspace_size(_params())
    Q = torch.empty(1, 24, 118800, 128, dtype=torch.bfloat16)
    big = spr.sparsepr_workspace_size(spr.make_params(Q, Ms=2048, p=32, Gk=256, Gq=256, M=1024,
                                                      r=32, route_mode="budget"))
    assert big > 20 * small
    assert big < 8e9  # fits easily in 180 GB


def test_noalloc_rejects_on_the_host(lib):
    f = lib.sparsepr_attend_routed_noalloc
    ok = dict(BH=2, N=4096, d=128, Gq=64, Gk=64)

    def call(ptr=256, runs=256, O=256, status=None, **kw):
        a = dict(ok, **kw)
        return f(ptr, ptr, ptr, 256, 256, runs, a["BH"], a["N"], a["d"], a["Gq"], a["Gk"], 0.0, O,
                 status, None)

    assert call(ptr=None) == spr._binding.SPR_EINVAL
    assert call(O=None) == spr._binding.SPR_EINVAL
    assert call(Gq=0) == spr._binding.SPR_EINVAL
    assert call(Gk=257) == spr._binding.SPR_EINVAL
    assert call(d=96) == spr._binding.SPR_EUNSUPPORTED
    assert call(ptr=264) == spr._binding.SPR_EUNSUPPORTED  # Q/K/V not 16-byte aligned
    assert call(runs=260) == spr._binding.SPR_EUNSUPPORTED  # ranges not 8-byte aligned
    # 256 + 80*BH (to 256) + 16*(BH*(ceil(N/128) + Gq) + 1) bytes must fit in 4 MiB
    assert call(BH=64, N=1 << 20, Gq=256) == spr._binding.SPR_ESCRATCH
    assert call(BH=40, N=75600, Gq=257) == spr._binding.SPR_EINVAL
