"""Derives the polynomial the attention kernel uses for part of its 2^x.

Method: Cody-Waite style range reduction x = n + f with n = round(x),
f in [-1/2, 1/2], so 2^x = 2^n * 2^f; 2^n is built by adding n to the float
exponent field, and 2^f is approximated by a degree-3 polynomial p(f) whose
coefficients minimise the maximum RELATIVE error on [-1/2, 1/2] (a minimax
fit computed here with a plain Remez exchange, the textbook algorithm).

The result only has to feed bf16 probabilities (8-bit mantissa, relative
step 2^-8) and an fp32 running sum, so a max relative error near 1e-4 is
ample.  Run this file to print the coefficients and the achieved error:

    python -m sliding_window_gqa_cu_b200.fit_exp2_poly
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _rel_err(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    return np.polynomial.polynomial.polyval(f, c) / np.exp2(f) - 1.0


def remez_exp2(degree: int = DEGREE, iters: int = 30) -> tuple[np.ndarray, float]:
    """Minimax (relative error) polynomial for 2^f on [LO, HI]; returns
    (coefficients c0..c_degree in increasing order, max relative error)."""
    n = degree + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    c = np.zeros(degree + 1)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :degree + 1] = xi ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * np.exp2(xi)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:degree + 1]
        e = _rel_err(c, grid)
        # new reference: one extremum of the error in each sign-alternating run
        sign = np.sign(e)
        bounds = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(grid.size), bounds)
        ext = [r[np.argmax(np.abs(e[r]))] for r in runs if r.size]
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        while len(ext) > n:
            drop = 0 if abs(e[ext[0]]) < abs(e[ext[-1]]) else len(ext) - 1
            ext.pop(drop)
        x = grid[np.array(ext)]
    err = float(np.max(np.abs(_rel_err(c, grid))))
    return c, err


def coefficients_f32() -> tuple[list[float], float]:
    c, _ = remez_exp2()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 200001).astype(np.float32)
    # error of the fp32 Horner evaluation actually used on the GPU
    p = np.float32(c32[3])
    for ci in c32[2::-1]:
        p = p * grid + np.float32(ci)
    err = float(np.max(np.abs(p.astype(np.float64) / np.exp2(grid.astype(np.float64)) - 1.0)))
    return [float(v) for v in c32], err


if __name__ == "__main__":
    coeffs, err = coefficients_f32()
    for i, v in enumerate(coeffs):
        print(f"c{i} = {v!r:>24}  ({np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error (fp32 Horner on [-1/2, 1/2]): {err:.3e}")
