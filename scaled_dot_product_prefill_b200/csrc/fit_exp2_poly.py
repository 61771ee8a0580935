"""Fit the degree-3 polynomial used by exp2_fma2 (sm100_ptx.cuh).

Minimises the maximum relative error of p(f) ~ 2^f on [-1/2, 1/2] with
Lawson's algorithm (iteratively reweighted least squares converging to the
minimax solution), then reports the error of the float32 coefficients
evaluated in float32 Horner form.  Run: python fit_exp2_poly.py
"""
import numpy as np


def fit(deg=3, iters=200):
    f = 0.5 * np.cos(np.linspace(0.0, np.pi, 4001))
    y = 2.0 ** f
    A = np.vander(f, deg + 1, increasing=True) / y[:, None]   # relative-error design matrix
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        err = np.abs(A @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_error_f32(c):
    x = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    acc = np.full_like(x, c[-1])
    for k in range(len(c) - 2, -1, -1):
        acc = (acc * x + c[k]).astype(np.float32)
    return float(np.max(np.abs(acc.astype(np.float64) / 2.0 ** x.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", [repr(float(v)) for v in c])
    print("max relative error (float32 Horner):", max_rel_error_f32(c))
