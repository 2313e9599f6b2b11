"""Coefficients of the FMA-pipe exp2 used by the prefill softmax.

Method (Cody & Waite style range reduction, 1980): 2^x = 2^n * 2^f with
n = round-to-nearest(x) and f = x - n in [-1/2, 1/2].  2^f is approximated by
a cubic p(f) fitted by least squares on 4096 Chebyshev nodes of [-1/2, 1/2] (a
near-minimax fit), with p(0) pinned to 1 so that integer powers of two are
exact.  Run this file to print the coefficients and the fit's maximum relative
error; prefill_tc.cu carries the printed values.
"""
import numpy as np


def fit(degree=3, nodes=4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    # p(f) = 1 + c1 f + c2 f^2 + c3 f^3: least squares on the relative error
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    coeffs = np.concatenate([[1.0], c]).astype(np.float32)
    ff = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(coeffs[::-1].astype(np.float64), ff)
    err = np.abs(p / np.exp2(ff) - 1).max()
    return coeffs, err


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}f" for v in c))
    print("max relative error on [-1/2, 1/2]:", err)
