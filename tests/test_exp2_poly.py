"""The polynomial 2^x of the attention softmax: its coefficients are the ones
the fit in free_block_sparse_means_b200/exp2_fit.py produces, and the kernel's
fp32 steps (mirrored in numpy) stay within 1e-4 relative of 2^x over the whole
range the softmax uses (x in [-125, 0]; smaller x is clamped), with exact
powers of two handled by the exponent step.  The kernel applies it to full
tiles only, so no masked key (-inf) reaches it."""
import os
import re

import numpy as np

from free_block_sparse_means_b200 import exp2_fit

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "free_block_sparse_means_b200", "csrc", "k_attend_tc.cu")


def _kernel_constants():
    text = open(SRC).read()
    vals = dict(re.findall(r"EXP2_C(\d) = ([0-9.eE+-]+)f", text))
    return np.array([float(vals[str(i)]) for i in range(4)])


def test_kernel_constants_are_the_fit():
    np.testing.assert_allclose(_kernel_constants(), exp2_fit.fit(), rtol=0, atol=2e-9)


def test_relative_error_over_the_softmax_range():
    c = _kernel_constants()
    assert exp2_fit.max_relative_error(c) < 1e-4
    x = np.float32(-np.linspace(0.0, 125.0, 1_000_001))
    got = exp2_fit.exp2_fp32(x, c).astype(np.float64)
    rel = np.abs(got / 2.0 ** x.astype(np.float64) - 1.0)
    assert rel.max() < 1e-4
    # integer arguments: 2^n exactly scaled from p(0)
    n = np.arange(0, -126, -1, dtype=np.float32)  # 0 .. -125
    np.testing.assert_allclose(exp2_fit.exp2_fp32(n, c) / 2.0 ** n.astype(np.float64),
                               np.float32(c[0]), rtol=1e-7)


def test_below_range_is_tiny_and_positive():
    c = _kernel_constants()
    got = exp2_fit.exp2_fp32(np.float32([-125.5, -200.0, -1e30]), c)
    assert (got > 0).all() and (got < 2.0 ** -124).all()
