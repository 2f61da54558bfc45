"""Derives the coefficients of the degree-3 polynomial that attn_tc.cu uses for 2^f on
f in [-0.5, 0.5] (the software exponential that takes part of the softmax's exponentials off the
special-function unit). Method: Cody-Waite style range reduction x = n + f, n = round(x), then a
minimax-style fit of 2^f in relative error by iteratively reweighted least squares; the
coefficients are rounded to float32 and the float32 Horner evaluation is checked.

    python paired_heads_b200/csrc/exp2_poly_fit.py
"""
import numpy as np


def fit(deg: int = 3, iters: int = 60):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    w = 1.0 / y
    for _ in range(iters):
        A = np.vander(f, deg + 1, increasing=True) * w[:, None]
        c, *_ = np.linalg.lstsq(A, y * w, rcond=None)
        err = (np.vander(f, deg + 1, increasing=True) @ c - y) / y
        w = w * (1 + 5 * np.abs(err) / np.abs(err).max())
    c32 = c.astype(np.float32)
    ff = f.astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) - y) / y
    return c32, float(rel.max())


if __name__ == "__main__":
    c, err = fit()
    print("coefficients c0..c3:", [float(x) for x in c])
    print("max relative error of the float32 evaluation: %.2e" % err)
