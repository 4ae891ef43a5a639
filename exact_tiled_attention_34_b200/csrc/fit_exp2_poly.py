"""Fit the coefficients of the cubic used for 2^f, f in [-1/2, 1/2], in fa_ptx.cuh.

    python exact_tiled_attention_34_b200/csrc/fit_exp2_poly.py

p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (constant term fixed at 1 so that 2^0 is exact),
fitted to minimise the maximum relative error |p(f) / 2^f - 1| over [-1/2, 1/2] by
iteratively reweighted least squares on a dense Chebyshev grid, then rounded to
float32. Prints the coefficients and the error bound measured in float64 on a
uniform grid of 2e5 points. Only NumPy is used; nothing here runs at build time.
"""
import numpy as np


def fit(iters: int = 80):
    f = 0.5 * np.cos(np.linspace(0.0, np.pi, 4001))
    y = np.exp2(f)
    w = np.ones_like(f)
    for _ in range(iters):
        # unknowns c1..c3; relative residual (1 + sum c_k f^k) / y - 1
        A = np.stack([f, f ** 2, f ** 3], axis=1) / y[:, None]
        b = 1.0 - 1.0 / y
        c, *_ = np.linalg.lstsq(A * w[:, None], b * w, rcond=None)
        err = (1.0 + np.stack([f, f ** 2, f ** 3], axis=1) @ c) / y - 1.0
        w = w * (1.0 + 50.0 * np.abs(err) / np.max(np.abs(err)))
        w /= w.mean()
    return np.float32(c)


def max_rel_err(c) -> float:
    g = np.linspace(-0.5, 0.5, 200001)
    p = 1.0 + g * (np.float64(c[0]) + g * (np.float64(c[1]) + g * np.float64(c[2])))
    return float(np.max(np.abs(p / np.exp2(g) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("c1 = %.9ef, c2 = %.9ef, c3 = %.9ef" % tuple(float(x) for x in c))
    print("max relative error on [-1/2, 1/2]: %.3e (2^%.2f)" % (max_rel_err(c), np.log2(max_rel_err(c))))
