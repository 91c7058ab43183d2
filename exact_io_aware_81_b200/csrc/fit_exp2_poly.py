"""Fit the polynomial used by the FMA-pipe exp2 in the prefill softmax.

2^x is evaluated as 2^j * q(f) with j = round(x) and f = x - j in [-1/2, 1/2]; q is a
polynomial with q(0) = 1 exactly (so that 2^-127 * q(0) packs to exactly +0 for masked
scores).  The remaining coefficients minimise the maximum relative error
|q(f) / 2^f - 1| on [-1/2, 1/2], found with Lawson's iteratively reweighted least squares
(an approximation of the minimax/Remez solution) on a dense grid, in float64.

Run:  python fit_exp2_poly.py [degree]   -- prints the coefficients c1..cn and the error
(the kernels use degree 4).
"""
import sys

import numpy as np


def fit(degree: int, iters: int = 200, n: int = 4001):
    f = np.linspace(-0.5, 0.5, n)
    target = np.exp2(f)
    # unknowns c1..cn of q(f) = 1 + sum_k c_k f^k, relative residual (q - 2^f) / 2^f
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target
    w = np.full(n, 1.0 / n)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * r
        s = w.sum()
        if s == 0:
            break
        w /= s
    q = 1.0 + sum(c[k - 1] * f ** k for k in range(1, degree + 1))
    err = np.max(np.abs(q / target - 1.0))
    return c, err


def max_error_float32(c):
    """Relative error of the float32 evaluation (Horner with fused multiply-adds)."""
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    q = np.float32(c[-1])
    for ck in reversed(c[:-1]):
        q = (q * f + np.float32(ck)).astype(np.float32)
    q = (q * f + np.float32(1.0)).astype(np.float32)
    return float(np.max(np.abs(q.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, err = fit(deg)
    for k, ck in enumerate(c, start=1):
        print(f"c{k} = {np.float32(ck)!r}  ({ck:.12e})")
    print(f"max relative error (float64 evaluation): {err:.3e}")
    print(f"max relative error (float32 evaluation): {max_error_float32([np.float32(x) for x in c]):.3e}")
