"""Fit the polynomial the attention kernel uses to compute part of its exponentials on the
FMA pipe instead of the MUFU.

Method (Cody & Waite, "Software Manual for the Elementary Functions", 1980: argument
reduction before a polynomial): 2^x = 2^j * 2^f with j = round(x) and f = x - j in
[-1/2, 1/2]; 2^j is applied by adding j to the exponent field, and 2^f by a degree-3
polynomial fitted here by iterated re-weighted least squares toward the minimax relative
error on [-1/2, 1/2] (Chebyshev nodes, Lawson's algorithm).

    python -m prefix_shared_attention_b200.csrc.fit_exp2_poly

prints the coefficients (float32, c0..c3) and the max relative error.  The kernel's
constants must equal this output (tests/test_exp2_poly.py checks it).
"""

from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, n: int = 4001, iters: int = 200):
    k = np.arange(n)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / n)            # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones(n) / n
    for _ in range(iters):                              # Lawson: w <- w * |relative error|
        sw = np.sqrt(w)[:, None]
        c, *_ = np.linalg.lstsq(V * sw / y[:, None], np.sqrt(w), rcond=None)
        err = np.abs(V @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    return c.astype(np.float32)


def max_rel_error(c: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 200001)
    p = np.polyval(np.asarray(c, np.float64)[::-1], f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("c0..c3 =", ", ".join(f"{v:.9e}f" for v in c))
    print("max relative error on [-1/2, 1/2]:", max_rel_error(c))
