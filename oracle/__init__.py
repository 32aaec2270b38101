"""CPU oracle for the SparsePR sparse attention call.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  The product path
(the CUDA library and its Python binding) never imports it and has no CPU
fallback.

Every function is a plain fp64 restatement of one step of the method as the
pages describe it; see ``sparsepr_oracle`` for the citations and readings.
Parity status: all functions are pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` (closed forms, brute force, invariants, library
routines on special cases).  The fit's internal U_r and B on the synthetic
workloads are "parity unpinned" when the probe residual is below 1e-3 of the
dense output in relative Frobenius norm; the final output is always compared.
"""
from .sparsepr_oracle import *  # noqa: F401,F403
from .sparsepr_oracle import __all__  # noqa: F401
