"""Fit the polynomial the softmax uses to evaluate 2^f on the FMA pipe.

Method: Remez exchange (minimax) for the RELATIVE error of a degree-n
polynomial p(f) ~ 2^f on f in [-1/2, 1/2], i.e. minimise max |p(f) 2^-f - 1|.
The kernel splits x = n + f with n = round(x), so 2^x = p(f) * 2^n exactly up
to p's error.  Coefficients are then rounded to fp32 and the fp32 Horner
evaluation is checked on a dense grid.

Run:  python fit_exp2_poly.py [degree]   (prints C initialisers)
"""
import sys

import numpy as np


def remez_relative(degree, lo=-0.5, hi=0.5, iters=30):
    n = degree
    # start from Chebyshev extrema
    k = np.arange(n + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - g(x_i) = (-1)^i E g(x_i)  (relative error equioscillation)
        g = np.exp2(x)
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * g[i]
        sol = np.linalg.solve(A, g)
        coef = sol[:n + 1]
        err = np.polyval(coef[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: one extremum per sign-alternating segment
        sign = np.sign(err)
        idx = np.flatnonzero(np.diff(sign) != 0)
        bounds = np.concatenate(([0], idx + 1, [len(grid)]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n + 2:
            break
        x = grid[ext]
    return coef


def fp32_eval(coef32, f):
    f = f.astype(np.float32)
    acc = np.float32(coef32[-1])
    for c in coef32[-2::-1]:
        acc = (acc * f + np.float32(c)).astype(np.float32)
    return acc


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    coef = remez_relative(degree)
    coef32 = np.array(coef, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 1000001)
    rel = np.abs(fp32_eval(coef32, f).astype(np.float64) / np.exp2(f) - 1.0).max()
    print("// degree %d, max relative error %.3e (fp32 Horner on [-1/2, 1/2])" % (degree, rel))
    for i, c in enumerate(coef32):
        print("constexpr float kExp2C%d = %.9ef;" % (i, float(c)))


if __name__ == "__main__":
    main()
