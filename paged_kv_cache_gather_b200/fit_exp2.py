"""Fit the polynomial behind the library's FMA-pipe exp2 (a building block for
taking softmax exponentials off the MUFU unit).

2^x is split exactly (Cody and Waite's range reduction, here in base 2 where it
is exact): x = j + f with j = round(x) and f in [-1/2, 1/2], so
2^x = 2^j * 2^f. The integer part goes straight into the exponent field; 2^f
is a cubic fitted here for minimum maximum *relative* error on [-1/2, 1/2] by
Lawson's iteratively reweighted least squares (which converges to the
minimax fit), in float64, then rounded to float32.

Run ``python -m paged_kv_cache_gather_b200.fit_exp2`` to print the
coefficients and their error bound; the kernel carries the printed values.
"""

import numpy as np


def fit(degree=3, iters=200, n=20001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones(n) / n
    c = None
    for _ in range(iters):
        sw = np.sqrt(w) / y  # relative error weighting
        c, *_ = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    # error of the float32 coefficients evaluated in float64 (Horner)
    p = np.zeros_like(f)
    for k in range(degree, -1, -1):
        p = p * f + np.float64(c32[k])
    rel = np.max(np.abs(p - y) / y)
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    print("coefficients (c0..c3):", ", ".join(f"{float(x):.9e}f" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {rel:.3e}")
