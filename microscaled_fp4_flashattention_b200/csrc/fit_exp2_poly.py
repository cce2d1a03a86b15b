"""Fit the polynomials 2^f ~ c0 + c1 f + ... on [0, 1) of the FMA-pipe exponentials:
degree 3 for ex2_poly2 in attn_fwd.cu (its result feeds E2M1 rounding) and degree 4 for
vl_ex2_fma2 in vlines.cu (column masses, relative error 2.7e-6).

Minimax in relative error by Lawson's algorithm (iteratively reweighted least squares on a
dense grid), then rounded to float32.  Prints the coefficients and the maximum relative error
of the float32 Horner evaluation.  Run: python fit_exp2_poly.py
"""
import numpy as np


def fit(deg: int = 3, n: int = 20001, iters: int = 2000):
    f = np.linspace(0.0, 1.0, n)
    target = 2.0 ** f
    a = np.vander(f, deg + 1, increasing=True) / target[:, None]   # rows: f^k / 2^f
    w = np.ones_like(f)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(a * np.sqrt(w)[:, None], np.sqrt(w), rcond=None)
        e = np.abs(a @ c - 1.0)
        w = w * e
        w /= w.sum()
    c32 = c.astype(np.float32)
    ff = f.astype(np.float32)
    p = np.full_like(ff, c32[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    return c32, float(np.max(np.abs(p.astype(np.float64) / target - 1.0)))


if __name__ == "__main__":
    for deg in (3, 4):
        c, err = fit(deg)
        print(f"degree {deg} coefficients (c0..c{deg}):", ", ".join(repr(float(x)) for x in c))
        print("  max relative error on [0, 1): %.3e" % err)
