"""Coefficients of the polynomial part of the forward kernel's FMA-pipe exp2.

The forward softmax computes 2^x for x <= 8 (x = lambda * s - m in log2
units). Part of those exponentials run on the FMA pipe instead of the
special-function unit, by Cody and Waite's range reduction (W. J. Cody and
W. Waite, "Software Manual for the Elementary Functions", 1980): x = n + f
with n = round(x) and f in [-1/2, 1/2], so 2^x = 2^n * 2^f, where 2^f comes
from a polynomial and 2^n is added into the exponent field.

This script finds the degree-3 polynomial with the smallest maximum relative
error on [-1/2, 1/2] by the Remez exchange algorithm (E. Ya. Remez, 1934),
rounds its coefficients to fp32, and checks the rounded polynomial's error
evaluated in fp32 arithmetic (Horner form, one rounding per fused
multiply-add, as the kernel does). `python exp2_poly.py` prints the
coefficients as they appear in fa_fwd.cuh; tests/test_exp2_poly.py checks
that the two agree and that the error bound holds.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _error(c, x):
    """Relative error of the polynomial with coefficients c (c[0] + c[1] x + ...)."""
    p = np.polynomial.polynomial.polyval(x, c)
    t = np.exp2(x)
    return (p - t) / t


def remez(degree: int = DEGREE, iters: int = 30):
    """Minimax (relative error) polynomial for 2^x on [LO, HI], float64."""
    n = degree + 2
    # Start from Chebyshev extrema mapped to the interval.
    k = np.arange(n)
    ref = 0.5 * (LO + HI) - 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  sum_j c_j x_i^j - (-1)^i 2^x_i E = 2^x_i
        A = np.zeros((n, n))
        for j in range(degree + 1):
            A[:, j] = ref ** j
        A[:, degree + 1] = -((-1.0) ** k) * np.exp2(ref)
        sol = np.linalg.solve(A, np.exp2(ref))
        c = sol[:degree + 1]
        err = _error(c, grid)
        # New reference: the extremum of |err| inside each run of equal sign.
        sign = np.sign(err)
        runs = np.flatnonzero(np.diff(sign) != 0) + 1
        bounds = np.concatenate([[0], runs, [len(grid)]])
        pts = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            i = a + int(np.argmax(np.abs(err[a:b])))
            pts.append(grid[i])
        if len(pts) != n:
            break
        new = np.array(pts)
        if np.max(np.abs(new - ref)) < 1e-15:
            ref = new
            break
        ref = new
    return c


def fp32_coefficients():
    return [float(np.float32(x)) for x in remez()]


def fp32_eval(c32, x):
    """The kernel's evaluation: Horner with fp32 fused multiply-adds."""
    x = np.asarray(x, dtype=np.float32)
    acc = np.full_like(x, np.float32(c32[-1]))
    for cj in reversed(c32[:-1]):
        # fp32 FMA: exact product and sum in float64, one rounding to fp32.
        acc = (acc.astype(np.float64) * x.astype(np.float64) + np.float64(np.float32(cj))).astype(np.float32)
    return acc


def max_rel_error_fp32(c32, samples: int = 1 << 20):
    x = np.linspace(LO, HI, samples, dtype=np.float32)
    p = fp32_eval(c32, x).astype(np.float64)
    t = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(p - t) / t))


if __name__ == "__main__":
    c32 = fp32_coefficients()
    for j, cj in enumerate(c32):
        print(f"c{j} = {np.float32(cj)!r}  ({np.float32(cj).view(np.uint32):#010x})")
    print(f"max relative error, fp32 Horner on [-1/2, 1/2]: {max_rel_error_fp32(c32):.3e}")
