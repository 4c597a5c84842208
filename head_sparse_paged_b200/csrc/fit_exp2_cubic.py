"""Fits the cubic p(f) ~ 2^f, f in [0, 1), that the prefill kernel evaluates on the FMA pipe for part of its
exponentials.

2^x is split as 2^n * 2^f with n = floor(x) and f = x - n (Cody-Waite range reduction); 2^n is applied by adding n
to the exponent bits, so only 2^f on [0, 1) needs a polynomial. The cubic minimises the maximum relative error
on a dense grid, posed as a linear program: minimise E subject to |p(f_i) - 2^f_i| <= E * 2^f_i. The kernel
rounds every probability to bf16 (relative step 2^-8) next, so an error near 1e-4 is immaterial.

Run: python head_sparse_paged_b200/csrc/fit_exp2_cubic.py -> the float32 coefficients (c0..c3, hex and decimal)
and the error of their float32 Horner evaluation.
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg: int = 3, n: int = 4001):
    f = np.linspace(0.0, 1.0, n)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)                  # columns f^0 .. f^deg
    # variables (c_0..c_deg, E): minimise E with  V c - y <= E y  and  y - V c <= E y
    cost = np.zeros(deg + 2)
    cost[-1] = 1.0
    a_ub = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b_ub = np.concatenate([y, -y])
    res = linprog(cost, A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * (deg + 1) + [(0, None)], method="highs")
    assert res.success, res.message
    return res.x[:-1], res.x[-1]


def horner32(c32, f32):
    p = np.float32(c32[-1])
    for ci in c32[-2::-1]:
        p = (p * f32 + ci).astype(np.float32)
    return p


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    f = np.linspace(0.0, 1.0, 1000001, endpoint=False).astype(np.float32)
    rel = np.abs(horner32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    print("c0..c3 (float32):", [float(v).hex() for v in c32], [repr(float(v)) for v in c32])
    print(f"max relative error: {e:.3e} (fit), {rel.max():.3e} (float32 Horner on [0, 1))")
