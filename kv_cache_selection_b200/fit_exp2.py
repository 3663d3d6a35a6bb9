"""Derivation of the polynomial in the library's FMA-pipe exponential
(exp2_fma in csrc/tc_common.cuh).

2^x = 2^j * 2^f with j = round(x) and f in [-1/2, 1/2].  The degree-3
polynomial p(f) ~ 2^f minimises the maximum relative error |p(f)/2^f - 1| on
[-1/2, 1/2]; it is computed with Lawson's algorithm (iteratively reweighted
least squares, C. L. Lawson, 1961), starting from uniform weights on a dense
grid.  Run `python -m kv_cache_selection_b200.fit_exp2` to print the float32
coefficients (constant term first) and the error of their float32 Horner
evaluation.
"""

from __future__ import annotations

import numpy as np


def fit(deg: int = 3, n: int = 20001, iters: int = 200):
    f = np.linspace(-0.5, 0.5, n)
    y = 2.0 ** f
    w = np.ones_like(f)
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        W = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = (V @ c - y) / y
        w = w * np.abs(err)
        w /= w.sum()
    c32 = c.astype(np.float32)
    ff = f.astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(deg - 1, -1, -1):
        p = p * ff + c32[k]
    rel = float(np.max(np.abs(p.astype(np.float64) - y) / y))
    return [float(x) for x in c32], rel


if __name__ == "__main__":
    coeffs, rel = fit()
    print("coefficients (f^0 .. f^3):", coeffs)
    print(f"max relative error of the float32 Horner form on [-1/2, 1/2]: {rel:.3e}")
