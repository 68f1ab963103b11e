"""Coefficients of the FMA-pipe 2^f polynomial used by the paired attention
kernel (attention_pair.cu) for part of its exponentials.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by a degree-4 polynomial whose coefficients minimise the
relative error sum((P(f) - 2^f) / 2^f)^2 over 4000 Chebyshev nodes of
[-1/2, 1/2] (weighted linear least squares), then rounded to fp32.  Prints
the coefficients and the worst relative error of the fp32-rounded polynomial
over a dense grid.  Run: python exp2_poly_fit.py
"""
import numpy as np


def fit(deg: int = 4, nodes: int = 4000):
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)
    w = 1.0 / np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True) * w[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones(nodes), rcond=None)
    return c.astype(np.float32)


def worst_rel_err(c):
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(f)
    for k in range(len(c) - 1, -1, -1):
        p = p * f + float(c[k])
    return float(np.abs(p / np.exp2(f) - 1).max())


if __name__ == "__main__":
    c = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f  // {v.view(np.uint32):#010x}")
    print("max relative error", worst_rel_err(c))
