"""Fit the polynomial the attention kernel uses to evaluate 2^f on the FMA
pipe for part of the softmax weights.

Method: for f in [0, 1), approximate 2^f by p(f) = 1 + c1 f + c2 f^2 + c3 f^3
(p(0) = 1 exactly, so a score equal to the running maximum gets weight
exactly 1).  The coefficients minimise the maximum RELATIVE error on a dense
grid of [0, 1] - a minimax fit solved as a linear program (minimise t
subject to |p(f_i) - 2^f_i| <= t 2^f_i).  Together with the split
x = j + f, j = floor(x), 2^x = p(f) * 2^j (the integer part goes straight
into the exponent field), this gives 2^x to about 1e-4 relative error,
below the bf16 rounding (2^-9) the weights get anyway.

Run: python fit_exp2_poly.py  -> prints the coefficients as fp32 literals.
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree: int = 3, n: int = 4001):
    f = np.linspace(0.0, 1.0, n)
    y = np.exp2(f)
    # variables: c1..c_deg, t ; minimise t
    A, b = [], []
    for fi, yi in zip(f, y):
        row = [fi ** k for k in range(1, degree + 1)]
        # p - y <= t y   ->  sum c_k f^k - t y <= y - 1
        A.append(row + [-yi]); b.append(yi - 1.0)
        # y - p <= t y   -> -sum c_k f^k - t y <= 1 - y
        A.append([-r for r in row] + [-yi]); b.append(1.0 - yi)
    c = np.zeros(degree + 1); c[-1] = 1.0
    res = linprog(c, A_ub=np.array(A), b_ub=np.array(b), bounds=[(None, None)] * (degree + 1),
                  method="highs")
    assert res.success
    return res.x[:degree], res.x[-1]


if __name__ == "__main__":
    coef, err = fit()
    c32 = np.float32(coef)
    f = np.linspace(0, 1, 100001, dtype=np.float64)
    p = 1.0 + f * (float(c32[0]) + f * (float(c32[1]) + f * float(c32[2])))
    print("coefficients (fp32):", [float(x) for x in c32])
    print("fp32 literals:", ", ".join(f"{float(x):.9e}f" for x in c32))
    print("max relative error (fp64 evaluation of the fp32 coefficients):",
          float(np.max(np.abs(p / np.exp2(f) - 1.0))), "LP bound:", err)
