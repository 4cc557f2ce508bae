"""Fit the polynomial of the forward kernel's FMA-pipe exponential.

The softmax of the forward kernel computes part of its exponentials 2^x
without the MUFU unit: x = n + r with n = round(x) and r in [-1/2, 1/2]
(Cody and Waite's argument reduction), 2^r from a polynomial p(r), and n added
to the exponent field of p(r).  This script fits p: the degree-3 polynomial
that minimises the largest relative error |p(r) / 2^r - 1| over [-1/2, 1/2],
by the Remez exchange algorithm in float64, then rounds the coefficients to
float32 and reports the relative error of the rounded polynomial evaluated
the way the kernel evaluates it (float32 Horner steps with fused
multiply-adds).  Its output is the coefficient block of sta_common.cuh.

    python sparse_local_attention_b200/csrc/fit_exp2_poly.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, lo: float = LO, hi: float = HI, iters: int = 40):
    """Minimax coefficients (constant term first) of 2^r on [lo, hi] in
    relative error, and the levelled error."""
    n = degree + 2
    # start from the extrema of the Chebyshev polynomial of degree n - 1
    x = 0.5 * (lo + hi) - 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(lo, hi, 400001)
    coef, level = None, None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  at the n reference points
        a = np.zeros((n, n))
        a[:, : degree + 1] = x[:, None] ** np.arange(degree + 1)
        a[:, degree + 1] = (-1.0) ** np.arange(n) * np.exp2(x)
        sol = np.linalg.solve(a, np.exp2(x))
        coef, level = sol[: degree + 1], abs(sol[degree + 1])
        err = np.polynomial.polynomial.polyval(grid, coef) / np.exp2(grid) - 1.0
        # new reference: the extremum of each run of equal sign
        sign = np.sign(err)
        cut = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(grid.size), cut)
        ext = np.array([r[np.argmax(np.abs(err[r]))] for r in runs])
        if ext.size > n:  # keep the n largest, in order
            ext = np.sort(ext[np.argsort(-np.abs(err[ext]))[:n]])
        if ext.size == n:
            x = grid[ext]
    return coef, level


def kernel_exp2(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """2^x as the kernel computes it, in float32 (x clamped at -126, rounded
    to the nearest integer n by adding 1.5 * 2^23, r = x - n, Horner steps as
    fused multiply-adds, n added to the exponent field)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (x - (t - magic)).astype(np.float32)
    c = np.asarray(c, dtype=np.float32)

    def fma(a, b, d):  # one rounding, as the hardware's fused multiply-add
        return (a.astype(np.float64) * b.astype(np.float64) + d.astype(np.float64)).astype(np.float32)

    p = np.full_like(r, c[3])
    for k in (2, 1, 0):
        p = fma(p, r, np.full_like(r, c[k]))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def main():
    coef, level = remez()
    c32 = coef.astype(np.float32)
    xs = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    rel = np.abs(kernel_exp2(xs, c32).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    print(f"// degree-{DEGREE} minimax fit of 2^r on [{LO}, {HI}]: levelled relative error {level:.3e};")
    print(f"// float32 coefficients, float32 evaluation over x in [-126, 8]: max relative error {rel.max():.3e}")
    for k, v in enumerate(c32):
        print(f"constexpr float kExp2C{k} = {float(v)!r}f;")


if __name__ == "__main__":
    main()
