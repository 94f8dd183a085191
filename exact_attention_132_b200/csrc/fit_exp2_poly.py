"""Fit the polynomial the forward kernel uses to evaluate part of its exponentials
on the FMA pipe instead of the special-function unit.

Method (Cody-Waite range reduction + minimax polynomial):
    2^x = 2^n * 2^f,   n = rint(x),   f = x - n in [-1/2, 1/2]
2^f is approximated by p(f) = c0 + c1 f + ... + cD f^D whose coefficients minimise
the maximum RELATIVE error max |p(f) / 2^f - 1| on [-1/2, 1/2].  They are found by
the Remez exchange algorithm in float64 and then rounded to float32 (the kernel's
precision); the reported error is the measured error of the float32-coefficient,
float32-Horner evaluation against float64 2^f.

    python exact_attention_132_b200/csrc/fit_exp2_poly.py [--degree 3]

The printed coefficients are the constants kC0..kC3 of ex2_poly_pair in sm100_ptx.cuh.
"""
from __future__ import annotations

import argparse

import numpy as np


def remez_relative(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = degree + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef, E = None, None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for the coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef, E = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(sign))[0] + 1, [len(grid)]))
        ext = []
        for a, b in zip(idx[:-1], idx[1:]):
            seg = np.abs(err[a:b])
            ext.append(a + int(np.argmax(seg)))
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        while len(ext) > n:
            vals = [abs(err[e]) for e in ext]
            drop = 0 if vals[0] < vals[-1] else len(ext) - 1
            ext.pop(drop)
        x = grid[ext]
    return coef, abs(E)


def f32_horner_error(coef32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 1_000_001).astype(np.float32)
    acc = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        acc = (acc * f + c).astype(np.float32)   # float32 Horner, as the kernel does with FMA
    return float(np.max(np.abs(acc.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--degree", type=int, default=3)
    a = ap.parse_args()
    coef, e = remez_relative(a.degree)
    c32 = coef.astype(np.float32)
    print(f"degree {a.degree}: minimax relative error (float64 coefficients) {e:.3e}")
    print(f"float32 coefficients, float32 Horner: max relative error {f32_horner_error(c32):.3e}")
    for i, c in enumerate(c32):
        print(f"  c{i} = {float(c)!r}f   // {float(c).hex()}")


if __name__ == "__main__":
    main()
