"""Refits the cubic behind exp2_fma (fb_ptx.cuh): 2^f on [-1/2, 1/2] with p(0) = 1.

The coefficients c1..c3 of p(f) = 1 + c1 f + c2 f^2 + c3 f^3 minimise the largest
relative error |p(f) / 2^f - 1| over [-1/2, 1/2].  They are found by Lawson's
algorithm: least squares on Chebyshev points, each point's weight multiplied by its
residual after every solve, which converges to the minimax (equioscillating) fit.
Prints the coefficients and the error they reach in float64.
"""
import numpy as np


def fit(iters: int = 200, deg: int = 3):
    x = 0.5 * np.cos(np.linspace(0.0, np.pi, 4001))
    y = np.exp2(x)
    a = np.stack([x ** k for k in range(1, deg + 1)], 1) / y[:, None]  # relative residual of the free terms
    b = (y - 1.0) / y
    w = np.ones_like(x)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], b * sw, rcond=None)
        w = w * np.abs(a @ c - b)
        w /= w.sum()
    coef = np.concatenate([[1.0], c])
    xs = np.linspace(-0.5, 0.5, 200001)
    err = np.abs(np.polyval(coef[::-1], xs) / np.exp2(xs) - 1.0).max()
    return coef, err


if __name__ == "__main__":
    coef, err = fit()
    print("coefficients c0..c3:", ", ".join(repr(float(c)) for c in coef))
    print(f"max relative error on [-1/2, 1/2]: {err:.4e}")
