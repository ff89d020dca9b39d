"""Fit the cubic used by the kernels' FMA-pipe exp2 (csrc/ptx.cuh, exp2_poly2).

Method: 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f is
approximated by a degree-3 polynomial whose coefficients minimise the relative
error in the least-squares sense on Chebyshev nodes of [-1/2, 1/2] (a standard
near-minimax construction), with the constant term pinned so that 2^0 = 1
exactly. Prints the coefficients as C float literals and the achieved maximum
relative error; the values in ptx.cuh were produced by this script.

Run: python exact_attention_155_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def fit(degree=3, nodes=4097):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes of [-1/2, 1/2]
    target = np.exp2(f)
    # p(f) = 1 + c1 f + c2 f^2 + c3 f^3, relative residual (p - 2^f) / 2^f.
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / target[:, None]
    rhs = (target - 1.0) / target
    c, *_ = np.linalg.lstsq(A, rhs, rcond=None)
    coef = np.concatenate([[1.0], c])
    xs = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(coef[::-1], xs)
    rel = np.max(np.abs(p / np.exp2(xs) - 1.0))
    return coef.astype(np.float32), rel


if __name__ == "__main__":
    coef, rel = fit()
    for i, c in enumerate(coef):
        print(f"c{i} = {float(c):.9e}f")
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
