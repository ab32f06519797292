"""Coefficients of the polynomial that the kernels use for 2^f on f in [-1/2, 1/2].

The kernels evaluate part of their exponentials on the FMA pipe instead of the
MUFU unit: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2], 2^n
applied by adding n to the exponent field and 2^f by this polynomial.

Method: minimax approximation of the relative error by the Remez exchange
algorithm (Remez, 1934), started from Chebyshev nodes; the error is measured
in float64 on a dense grid. Run this script to regenerate the table printed
into exp2_poly.cuh; ``python gen_exp2_poly.py --check`` only verifies the
committed table's error bound.
"""
from __future__ import annotations

import os
import re
import sys

import numpy as np

DEGREE = 4
GRID = np.linspace(-0.5, 0.5, 200001)
HEADER = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exp2_poly.cuh")


def rel_err(c, f):
    return np.polynomial.polynomial.polyval(f, c) / np.exp2(f) - 1.0


def remez(deg: int, iters: int = 30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    x = 0.5 * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * np.exp2(xi)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        e = rel_err(c, GRID)
        # new reference: the extrema of each sign run of the error
        sign = np.sign(e)
        breaks = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(GRID.size), breaks)
        ext = [r[np.argmax(np.abs(e[r]))] for r in runs if r.size]
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        while len(ext) > n:
            if abs(e[ext[0]]) < abs(e[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = GRID[ext]
    return c, float(np.max(np.abs(rel_err(c, GRID))))


def committed():
    text = open(HEADER).read()
    vals = re.findall(r"kExp2Poly(\d) = ([-+0-9.eE]+)f;", text)
    c = np.zeros(len(vals))
    for i, v in vals:
        c[int(i)] = float(v)
    return c


def main():
    if "--check" in sys.argv:
        c = committed()
        err = float(np.max(np.abs(rel_err(c.astype(np.float32).astype(np.float64), GRID))))
        print(f"committed degree-{c.size - 1} table: max relative error {err:.3e}")
        return
    c, err = remez(DEGREE)
    print(f"// degree {DEGREE}, max relative error {err:.3e} on [-0.5, 0.5]")
    for i, v in enumerate(c):
        print(f"constexpr float kExp2Poly{i} = {float(np.float32(v))!r}f;")


if __name__ == "__main__":
    main()
