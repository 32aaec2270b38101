"""Coefficients of the polynomial 2^x used by the attention softmax for a share
of its exponentials (the rest go to the hardware approximation).

    python -m free_block_sparse_means_b200.exp2_fit

Method.  Cody & Waite's argument reduction: x = n + f with n = round(x), so
f lies in [-1/2, 1/2] and 2^x = 2^n * 2^f; 2^n is applied exactly by adding n
to the floating-point exponent field, 2^f comes from a polynomial.  The
polynomial minimises the maximum *relative* error on [-1/2, 1/2]: it is found
by iteratively reweighted least squares (Lawson's algorithm), starting from
least squares on Chebyshev nodes and multiplying each node's weight by its
current error, which drives the fit toward the equioscillating minimax
solution.  Degree 3 gives a relative error of 7.5e-5, well under the bf16
rounding (2^-9) the probabilities are stored with.

The kernel evaluates the same steps in fp32 (see exp2_poly in
csrc/k_attend_tc.cu); exp2_fp32 below mirrors them in numpy for the tests.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
MAGIC = np.float32(12582912.0)  # 1.5 * 2^23: adding it rounds to an integer


def fit(degree: int = DEGREE, iters: int = 60, nodes: int = 4001) -> np.ndarray:
    """Coefficients c_0 .. c_degree of p(f) ~ 2^f on [-1/2, 1/2] (relative error)."""
    f = 0.5 * np.cos(np.linspace(0.0, np.pi, nodes))
    y = 2.0 ** f
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        e = np.abs(A @ c - 1.0)
        w = w * (e / e.max() + 1e-3)
        w /= w.mean()
    return c


def exp2_fp32(x, c) -> np.ndarray:
    """The kernel's fp32 steps: clamp at -125 (the result stays a normal
    number), round by the magic constant, Horner in fp32, add n to the
    exponent field."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + MAGIC).astype(np.float32)
    f = (x - (t - MAGIC)).astype(np.float32)
    c = [np.float32(v) for v in c]
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def max_relative_error(c, n: int = 1 << 21, seed: int = 0) -> float:
    x = np.float32(-np.random.default_rng(seed).random(n) * 125.0)
    got = exp2_fp32(x, c).astype(np.float64)
    return float(np.abs(got / 2.0 ** x.astype(np.float64) - 1.0).max())


if __name__ == "__main__":
    c = fit()
    print("constexpr float " + ", ".join(f"EXP2_C{i} = {v:.9f}f" for i, v in enumerate(c)) + ";")
    print(f"max relative error in fp32: {max_relative_error(c):.2e}")
