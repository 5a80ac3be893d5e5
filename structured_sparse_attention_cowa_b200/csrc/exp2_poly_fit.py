"""Fit the cubic used by the kernels to compute 2^f on [0, 1) on the FMA pipe.

    python structured_sparse_attention_cowa_b200/csrc/exp2_poly_fit.py

Method: Lawson's algorithm (iteratively reweighted least squares converging to the
minimax solution) for the relative error |p(f) / 2^f - 1| on a dense grid of [0, 1],
in float64, then rounding the coefficients to float32.  The printed constants are the
ones in exp2_poly.cuh; tests/test_exp2_poly.py re-runs this fit and checks the header
and the error bound of the float32 evaluation.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, n_grid: int = 4001, iters: int = 400):
    f = np.linspace(0.0, 1.0, n_grid)
    target = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.full(n_grid, 1.0 / n_grid)
    c = None
    for _ in range(iters):
        # weighted LS in relative terms: minimise sum w * (p(f)/2^f - 1)^2
        A = V / target[:, None] * np.sqrt(w)[:, None]
        b = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A, b, rcond=None)
        err = np.abs(V @ c / target - 1.0)
        w = w * err
        s = w.sum()
        if s == 0:
            break
        w /= s
    return c


def eval_f32(coef32: np.ndarray, x: np.ndarray) -> np.ndarray:
    """The kernel's steps in float32: floor via x + (-magic) rounding, Horner, exponent add."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-120.0))
    n = np.floor(x).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.float32(coef32[3])
    for k in (2, 1, 0):
        p = (p * f + np.float32(coef32[k])).astype(np.float32)
    bits = p.view(np.int32) + (n.astype(np.int32) << 23)
    return bits.view(np.float32)


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    xs = np.linspace(-30.0, 8.0, 200001).astype(np.float32)
    rel = np.abs(eval_f32(c32, xs).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1.0)
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error of the float32 evaluation on [-30, 8]: {rel.max():.3e}")
