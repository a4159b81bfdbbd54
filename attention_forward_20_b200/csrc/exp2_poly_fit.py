"""Coefficients of the FMA-pipe exponential in sm100_ptx.cuh (exp2_fma2).

2^x is split as 2^j * 2^f with j = floor(x) and f = x - j in [0, 1); the
kernel puts j into the exponent field and evaluates 2^f with a polynomial
p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (Horner, fp32 FMAs).  p(0) = 1 exactly, so
an argument clamped to -127 gives exactly +0.0.

The coefficients minimise the largest relative error |p(f) / 2^f - 1| on
[0, 1] (a Remez exchange on the equioscillation conditions
p(f_i) - 2^f_i = (-1)^i E 2^f_i at deg + 1 reference points, with the
reference moved to the error's extrema until it settles).

python exp2_poly_fit.py     prints the float32 coefficients and the error.
"""
import numpy as np


def fit(deg=3, iters=40, grid_points=200001):
    """(c1..c_deg as float64, max relative error on [0, 1])."""
    n = deg
    grid = np.linspace(0.0, 1.0, grid_points)
    x = 0.5 - 0.5 * np.cos(np.pi * np.arange(n + 1) / n)  # Chebyshev-like start
    c = np.zeros(n)
    for _ in range(iters):
        a = np.zeros((n + 1, n + 1))
        rhs = np.zeros(n + 1)
        for i, xi in enumerate(x):
            t = 2.0 ** xi
            a[i, :n] = [xi ** (k + 1) for k in range(n)]
            a[i, n] = -((-1) ** i) * t
            rhs[i] = t - 1.0
        c = np.linalg.solve(a, rhs)[:n]
        err = evaluate(c, grid) / 2.0 ** grid - 1.0
        sign = np.sign(err)
        segments = np.split(np.arange(grid.size), np.where(np.diff(sign) != 0)[0] + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segments]
        while len(ext) > n + 1:
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        if len(ext) < n + 1:
            break
        x = grid[ext]
    err = evaluate(c, grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


def evaluate(c, f):
    p = np.zeros_like(f)
    for ck in c[::-1]:
        p = (p + ck) * f
    return p + 1.0


if __name__ == "__main__":
    c, e = fit()
    for k, ck in enumerate(c, 1):
        print(f"c{k} = {np.float32(ck)!r}")
    print(f"max relative error {e:.3e}")
