"""Fits the polynomial used for 2^f, |f| <= 1/2, in the kernels' FMA-pipe
exponential (range reduction x = n + f with n = round(x), then 2^x = 2^n * p(f)).

Minimax in relative error by Lawson's iteratively re-weighted least squares on
a dense grid; prints the coefficients (lowest degree first) and the error.
Run:  python exact_io_aware_55_b200/csrc/gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def fit(degree: int, iters: int = 200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        A = V * (w / y)[:, None]
        c, *_ = np.linalg.lstsq(A, w, rcond=None)
        err = np.abs(V @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32).astype(np.float64)
    err32 = np.max(np.abs(V @ c32 / y - 1.0))
    return c32, err32


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = fit(deg)
    print("coefficients:", ", ".join(f"{x:.9e}f" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e} (2^{np.log2(e):.1f})")
