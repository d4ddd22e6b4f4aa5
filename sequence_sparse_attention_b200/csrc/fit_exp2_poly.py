"""Coefficients of the polynomial the scoring kernel uses for 2^f on the FMA pipe.

    python fit_exp2_poly.py

Fits p(f) = c0 + c1 f + c2 f^2 + c3 f^3 + c4 f^4 to 2^f on [-1/2, 1/2] in
RELATIVE error by Lawson's iteratively reweighted least squares (the weights
converge to those of the minimax fit), rounds the coefficients to float32 and
reports the maximum relative error of the float32 Horner evaluation.  The
kernel reduces 2^a to 2^n * 2^f with n = round(a), f = a - n in [-1/2, 1/2].
"""
import numpy as np


def fit(deg=4, points=40001, iters=300):
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    A = np.vstack([f ** k for k in range(deg + 1)]).T
    w = np.ones_like(f)
    for _ in range(iters):
        W = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(A * W[:, None], y * W, rcond=None)
        e = np.abs(A @ c - y) / y
        w = w * e
        w /= w.sum()
    return np.float32(c)


def horner_f32(c, f):
    f = np.asarray(f, dtype=np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + np.float32(c[k])).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    f = np.linspace(-0.5, 0.5, 40001)
    err = np.max(np.abs(horner_f32(c, f).astype(np.float64) - np.exp2(f)) / np.exp2(f))
    print("coefficients c0..c4:", [repr(float(x)) for x in c])
    print("max relative error (fp32 Horner):", float(err))
