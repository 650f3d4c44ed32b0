"""Fit the polynomial exp2 used for part of the softmax in the attention kernel.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by a degree-4 polynomial in f, fitted here by weighted least
squares on 4096 Chebyshev nodes with weight 1/2^f (relative error), then
rounded to fp32. The printed coefficients are the ones in phase1_sm100.cu;
the fit and its error bound are re-checked by the CPU tests.

    python block_sparse_long_rope_b200/csrc/fit_exp2_poly.py
"""
import numpy as np

DEGREE = 4


def fit(degree=DEGREE, nodes=4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(f), rcond=None)
    return c.astype(np.float32)


def max_rel_error(c, samples=200001):
    f = np.linspace(-0.5, 0.5, samples)
    p = np.zeros_like(f)
    for a in c[::-1].astype(np.float64):
        p = p * f + a
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    for i, a in enumerate(c):
        print(f"c{i} = {float(a):.9e}f")
    print("max relative error on [-1/2, 1/2]:", max_rel_error(c))
