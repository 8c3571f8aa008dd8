"""Coefficients of the polynomial exp2 used by the attention forward.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(the argument reduction of Cody and Waite, "Software Manual for the
Elementary Functions", 1980, for base 2 the split needs no constant);
2^f is a polynomial whose coefficients this script fits by the Remez
exchange algorithm, minimising the largest relative error
|p(f) / 2^f - 1| over the interval.  The fit runs in float64, then the
coefficients are rounded to float32 and the error of the rounded
polynomial, evaluated in float32 by Horner's rule, is reported over a dense
grid.

    python -m folded_tensor_sequence_map_b200.csrc.fit_exp2 [degree]

prints the coefficients (c0 first) as C float literals and the error.
"""

from __future__ import annotations

import sys

import numpy as np

LO, HI = -0.5, 0.5


def remez_relative(degree: int, iters: int = 40) -> np.ndarray:
    """Minimax (relative error) polynomial for 2^f on [LO, HI]."""
    n = degree + 2
    # Chebyshev extrema as the first reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        # p(x_i) - (-1)^i E 2^x_i = 2^x_i  <=>  p(x_i)/2^x_i - 1 = (-1)^i E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign run of the error
        sign = np.sign(err)
        cuts = np.nonzero(np.diff(sign) != 0)[0] + 1
        runs = np.split(np.arange(len(grid)), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs if len(r)]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest magnitudes
        while len(ext) > n:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext.pop(drop)
        x_new = grid[ext]
        if np.allclose(x_new, x, atol=1e-12):
            break
        x = x_new
    return c


def horner_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """p(f) by Horner's rule, every step rounded to float32 (the kernel uses
    fused multiply-adds, whose single rounding is no worse)."""
    f = f.astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f + np.float64(ck)).astype(np.float32)
    return acc


def main(degree: int = 5) -> None:
    c = remez_relative(degree)
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 1000001)
    e64 = np.abs(np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0).max()
    e32 = np.abs(horner_f32(c32, grid).astype(np.float64) / 2.0 ** grid.astype(np.float32).astype(np.float64) - 1.0).max()
    for i, ck in enumerate(c32):
        print(f"c{i} = {float(ck).hex()}  /* {float(ck):.9e} */")
    print(f"max relative error: {e64:.3e} (float64 coefficients), {e32:.3e} (float32, Horner in float32)")


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else 5)
