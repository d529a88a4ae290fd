"""Coefficients of the kernels' polynomial exp2 (ptx.cuh, exp2_poly2).

exp2_poly2(z) splits z = j + f with j = rint(z) and f in [-1/2, 1/2], evaluates p(f) ~ 2^f with a
degree-5 polynomial in Horner form (float32 FMAs) and adds j to the exponent field.  The
coefficients minimise the maximum relative error max |p(f) / 2^f - 1| over [-1/2, 1/2]: the Remez
exchange algorithm (E. Ya. Remez, 1934) on the error function p(f) 2^-f - 1, run here in
float64, then rounded to float32.

Run as a script to print the coefficients in the form ptx.cuh holds them.
"""
from __future__ import annotations

import numpy as np

DEGREE = 5
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30) -> np.ndarray:
    """Minimax-relative-error polynomial for 2^f on [LO, HI]; coefficients c0..c_degree."""
    n = degree + 2
    # Chebyshev extrema as the first reference set
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    c = np.zeros(degree + 1)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i for the coefficients and the level E
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1.0) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(a, 2.0 ** x)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        idx = np.flatnonzero(np.diff(sign) != 0)
        bounds = np.concatenate(([0], idx + 1, [grid.size]))
        ext = [b0 + int(np.argmax(np.abs(err[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:])
               if b1 > b0]
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        while len(ext) > n:
            vals = np.abs(err[ext])
            drop = 0 if vals[0] < vals[-1] else len(ext) - 1
            ext.pop(drop)
        x = grid[ext]
    return c


def coefficients_f32() -> np.ndarray:
    return remez().astype(np.float32)


def eval_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """Horner evaluation with float32 FMAs (each FMA emulated exactly in float64 and rounded
    once to float32: a float32 product fits in float64)."""
    f = np.asarray(f, np.float32)
    acc = np.full(f.shape, c32[-1], np.float32)
    for ck in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return acc


if __name__ == "__main__":
    c = coefficients_f32()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  ({np.asarray(v).view(np.uint32):#010x})")
