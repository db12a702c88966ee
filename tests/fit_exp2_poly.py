"""Derives the cubic used by the prefill kernel to evaluate 2^f on the FMA
pipe for part of the softmax exponentials.

Method: range reduction x = n + f with n = round-to-nearest(x), f in
[-1/2, 1/2], so 2^x = 2^n * 2^f, where 2^n is applied by adding n to the
exponent field; 2^f is approximated by a degree-3 polynomial whose
coefficients minimise the maximum relative error on [-1/2, 1/2]. The
minimax fit uses Lawson's iteratively reweighted least squares on a dense
Chebyshev grid (float64).

Run as a script to print the coefficients in the form written into
ex2_poly (gqa_attention_rope_b200/csrc/ptx.cuh); tests/test_exp2_poly.py re-runs the fit and checks the
kernel's constants and the error bound.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, n_points: int = 4001, iters: int = 200):
    k = np.arange(n_points)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n_points)  # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative-error design matrix
    w = np.full(n_points, 1.0 / n_points)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(n_points) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def max_rel_error(c, n_points: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, n_points)
    return float(np.max(np.abs(np.polyval(c[::-1], f) / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients c0..c3:", ", ".join(f"{float(np.float32(x))!r}f" for x in c))
    print("max relative error (float64 evaluation):", max_rel_error(c))
