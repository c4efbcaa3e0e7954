"""Derives the coefficients of the degree-3 polynomial that attend.cuh uses for part of its exp2 work.

Method (Cody-Waite range reduction, then a minimax polynomial): write x = n + f with n = round(x) and
f in [-1/2, 1/2]; then 2^x = 2^n * 2^f, where 2^n is an exponent-field add and 2^f ~ p(f). The cubic p
minimises the maximum relative error on [-1/2, 1/2]; it is found here by iteratively reweighted least
squares on a dense grid (a Lawson-style approximation to the minimax fit), with p(0) left free.

P values feed a bf16 MMA (8 mantissa bits, relative spacing 2^-8 = 3.9e-3), so a relative error of a
few 1e-5 is far below the rounding that follows. Run: python gen_exp2_poly.py
"""
import numpy as np


def fit(degree=3, iters=60, n=20001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    w = np.ones_like(f)
    V = np.vander(f, degree + 1, increasing=True)
    for _ in range(iters):
        A = V / y[:, None] * np.sqrt(w)[:, None]
        b = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A, b, rcond=None)
        err = np.abs(V @ c / y - 1.0)
        w = w * (err / err.max() + 1e-3)
        w /= w.sum()
    c32 = c.astype(np.float32)
    err32 = np.abs((V @ c32.astype(np.float64)) / y - 1.0).max()
    return c32, err32


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  // {v.view(np.uint32):#010x}")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
