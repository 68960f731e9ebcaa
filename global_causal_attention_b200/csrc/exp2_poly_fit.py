"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2]
used by ptx.cuh's exp2_poly (the softmax evaluates part of its exponentials
on the FMA pipe; see the comment there).

Method: minimise the maximum relative error |p(f) / 2^f - 1| by iteratively
re-weighted least squares (Lawson's algorithm) on a dense grid, then round the
coefficients to float32 and report the error of the rounded polynomial.

    python exp2_poly_fit.py      ->  prints the float32 coefficients and the max error
"""
import numpy as np


def fit(deg=3, n=20001, iters=300):
    f = np.linspace(-0.5, 0.5, n)
    y = 2.0 ** f
    V = np.vander(f, deg + 1, increasing=True)
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V / y[:, None] * sw[:, None], sw, rcond=None)
        err = np.abs(V @ c / y - 1.0)
        w = w * (err / err.max() + 1e-12) ** 0.5
        w /= w.sum()
    c32 = c.astype(np.float32)
    err32 = float(np.abs(V @ c32.astype(np.float64) / y - 1.0).max())
    return c32, err32


if __name__ == "__main__":
    c, e = fit()
    print("coefficients (f32):", ", ".join(f"{float(x):.9g}f" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
