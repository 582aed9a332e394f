"""Fits the polynomial used to evaluate 2^f, f in [-1/2, 1/2], on the FMA
pipe (the attention softmax computes part of its exponentials this way
instead of on the special-function unit).

Method (range reduction by the nearest integer): 2^x = 2^n * 2^f with
n = round(x), f = x - n. The rounding is done with additions only: adding
1.5 * 2^23 to x leaves n in the low mantissa bits of the sum, subtracting it
again gives n as a float, and the scaling by 2^n is an integer add of n << 23
to the bits of 2^f. 2^f ~ 1 + c1 f + c2 f^2 + c3 f^3, the constant term fixed
at 1 so that 2^n is exact; c1..c3 minimise the maximum relative error on
[-1/2, 1/2] (a linear program on a dense grid), then are rounded to float32.

    python packed_attention_qk_b200/csrc/fit_exp2_poly.py
prints the coefficients and the relative error of the float32 evaluation.
"""

import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001, lo=-0.5, hi=0.5):
    f = np.linspace(lo, hi, n)
    y = np.exp2(f)
    # variables: c1..c_deg, t ; minimise t subject to |(1 + sum c_k f^k) / y - 1| <= t
    A = np.stack([f ** k / y for k in range(1, degree + 1)], axis=1)
    b = 1.0 - 1.0 / y
    ones = np.ones((n, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([b, -b])
    c = np.zeros(degree + 1)
    c[-1] = 1.0
    r = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * degree + [(0, None)], method="highs")
    return r.x[:degree], r.x[-1]


def eval_f32(coef, f):
    f = f.astype(np.float32)
    acc = np.float32(coef[-1])
    for c in coef[-2::-1]:
        acc = np.float32(acc * f + np.float32(c))
    return np.float32(acc * f + np.float32(1.0))


if __name__ == "__main__":
    coef, err = fit()
    c32 = [np.float32(c) for c in coef]
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float64)
    rel = np.abs(eval_f32(c32, f).astype(np.float64) / np.exp2(f) - 1.0)
    print("coefficients (c1, c2, c3):", [float(c) for c in c32])
    print("float32 hex:", [hex(np.float32(c).view(np.uint32)) for c in c32])
    print(f"minimax relative error {err:.3e}; float32 evaluation max {rel.max():.3e}")
