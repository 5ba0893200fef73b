"""Fit the cubic used for 2^f, |f| <= 1/2, in the kernels' FMA-pipe exp2.

Method: minimise the maximum relative error of c0 + c1 f + c2 f^2 + c3 f^3 against
2^f on [-1/2, 1/2] by iteratively reweighted least squares on Chebyshev nodes
(weights 1/2^f for relative error, Lawson's update towards the minimax solution).
Prints the coefficients as float32 literals and the achieved bound.
"""
import numpy as np


def fit(degree=3, nodes=4001, iters=200):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative-error system
    b = np.ones_like(f)
    w = np.full(nodes, 1.0 / nodes)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    fine = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(c32[::-1].astype(np.float64), fine) / np.exp2(fine) - 1).max()
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
