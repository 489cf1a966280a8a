"""Derives the coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on
f in [-1/2, 1/2] used by the prefill kernel's FMA-pipe exp2 (see exp2_fma in
ptx.cuh), by Lawson's iteratively reweighted least squares for the minimax
relative error (weights multiplied by the pointwise error each round), then
rounded to fp32.  Prints the coefficients and the max relative error of the
fp32 Horner evaluation over a dense grid.

Usage: python exp2_poly_fit.py [degree]
"""
import sys

import numpy as np


def fit(degree: int = 3, n: int = 4001, rounds: int = 200):
    f = np.cos(np.linspace(0, np.pi, n)) * 0.5          # Chebyshev-spaced nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative-error rows
    w = np.full(n, 1.0 / n)
    c = None
    for _ in range(rounds):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(n) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def horner_f32(c, f):
    c = [np.float32(x) for x in c]
    f = f.astype(np.float32)
    acc = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        acc = (acc * f + c[k]).astype(np.float32)
    return acc


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = fit(deg)
    grid = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(horner_f32(c, grid).astype(np.float64) / np.exp2(grid) - 1.0).max()
    for k, x in enumerate(c):
        print("c%d = %.9ef" % (k, np.float32(x)))
    print("max relative error (fp32 Horner): %.3e" % rel)
