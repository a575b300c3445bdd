"""Coefficients of the cubic used for 2^f, f in [0, 1), in the prefill softmax.

Part of the softmax exponentials run on the FMA pipe instead of the MUFU unit:
2^x = 2^floor(x) * 2^f with f = x - floor(x), and 2^f by a cubic.  The cubic
is fitted here by weighted least squares on Chebyshev nodes, minimising the
*relative* error (weight 1/2^f), with the two end values pinned exactly
(p(0) = 1, p(1) = 2) so that the pieces join continuously at integers.  The
result is rounded to fp32.  The maximum relative error (printed) is well below
the bf16 rounding of P (2^-9 = 1.95e-3) that follows.

Run:  python derive_exp2_poly.py
"""
import numpy as np


def fit(deg=3, n=4000):
    # Chebyshev nodes on [0, 1]
    k = np.arange(n)
    f = 0.5 - 0.5 * np.cos((2 * k + 1) * np.pi / (2 * n))
    y = np.exp2(f)
    w = 1.0 / y
    # p(f) = 1 + f * (c1 + c2 f + c3 f^2), with c1 + c2 + c3 = 1 (so p(1) = 2)
    # eliminate c1 = 1 - c2 - c3:  p - 1 - f = c2 (f^2 - f) + c3 (f^3 - f)
    A = np.stack([(f ** j - f) for j in range(2, deg + 1)], axis=1) * w[:, None]
    b = (y - 1.0 - f) * w
    c_hi, *_ = np.linalg.lstsq(A, b, rcond=None)
    c = np.concatenate([[1.0, 1.0 - c_hi.sum()], c_hi])
    c32 = c.astype(np.float32)
    xs = np.linspace(0, 1, 200001, dtype=np.float64)
    p = np.polyval(c32[::-1].astype(np.float64), xs)
    rel = np.abs(p / np.exp2(xs) - 1).max()
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}  ({v.view(np.uint32):#010x})")
    print(f"max relative error on [0,1): {rel:.3e}")
