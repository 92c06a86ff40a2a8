"""Coefficients of the polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on
f in [-1/2, 1/2], used by the softmax kernel to evaluate part of its
exponentials on the FMA pipe instead of the special-function unit.

Method: Cody-Waite style range reduction x = n + f with n = round(x) (so
2^x = 2^f * 2^n, the 2^n applied by adding n to the float's exponent field),
and a minimax fit of 2^f for *relative* error obtained with Lawson's algorithm
(iteratively reweighted least squares, C. L. Lawson 1961) on a dense grid.
Run ``python exp2_poly.py`` to print the float32 coefficients and the
maximum relative error of the float32 Horner evaluation.
"""
import numpy as np

DEGREE = 3


def fit(degree=DEGREE, n=20001, iters=400):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative-error design matrix
    w = np.full(n, 1.0 / n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], np.ones(n) * sw, rcond=None)
        err = np.abs(V @ c - 1.0)
        w = w * err
        w /= w.sum()
    return c


def horner_f32(c, f):
    c = np.asarray(c, np.float32)
    f = np.asarray(f, np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    rel = np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v)!r:>24}  ({v.view(np.uint32):#010x})")
    print(f"max relative error (float32 Horner): {rel.max():.3e}")
