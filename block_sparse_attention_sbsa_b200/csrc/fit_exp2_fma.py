"""Fits the polynomial of exp2_fma.cuh: 2^f on [-1/2, 1/2] by a degree-3
polynomial with the smallest largest relative error.

Method: Lawson's iteration (iteratively reweighted least squares, which
converges to the minimax fit) on 4001 Chebyshev points of the interval,
weighting each point by its relative error. Prints the coefficients c0..c3
(lowest degree first) rounded to float32, and the largest relative error of
the whole float32 evaluation (range reduction, Horner with fused
multiply-adds, exponent assembly) over x in [-125, 8], the range of the
softmax's arguments.

    python block_sparse_attention_sbsa_b200/csrc/fit_exp2_fma.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
ITERATIONS = 60
ROUND = np.float32(12582912.0)  # 1.5 * 2^23: x + ROUND rounds x to an integer


def fit(degree: int = DEGREE, iterations: int = ITERATIONS) -> np.ndarray:
    f = np.cos(np.linspace(0.0, np.pi, 4001))[::-1] * 0.5
    y = np.exp2(f)
    v = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    c = None
    for _ in range(iterations):
        a = v / y[:, None] * np.sqrt(w)[:, None]
        c, *_ = np.linalg.lstsq(a, np.sqrt(w), rcond=None)
        err = np.abs(v @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def fma32(a, b, c):
    """float32 fused multiply-add: the float64 product of two float32 values
    is exact, so one rounding of the float64 sum to float32 follows it
    (up to rare double rounding, far below the fit's error)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def eval32(c: np.ndarray, x: np.ndarray) -> np.ndarray:
    """The float32 steps of exp2_fma: clamp, Cody-Waite split x = n + f with
    n = round(x), Horner in fused multiply-adds, 2^n added to the exponent
    field, and 0 below -125."""
    x = x.astype(np.float32)
    xc = np.maximum(x, np.float32(-125.0))
    t = (xc + ROUND).astype(np.float32)
    n = (t - ROUND).astype(np.float32)
    f = (xc - n).astype(np.float32)
    q = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        q = fma32(q, f, np.full_like(f, c[k]))
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return np.where(x < np.float32(-125.0), np.float32(0.0), bits.view(np.float32))


def max_rel_error(c: np.ndarray, n: int = 2_000_000, seed: int = 0) -> float:
    x = np.random.default_rng(seed).uniform(-125.0, 8.0, n).astype(np.float32)
    exact = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(eval32(c, x) / exact - 1.0)))


if __name__ == "__main__":
    coef = fit()
    for k, v in enumerate(coef):
        print(f"c{k} = {float(v):.9e}f")
    print(f"largest relative error of the float32 evaluation: {max_rel_error(coef):.3e}")
