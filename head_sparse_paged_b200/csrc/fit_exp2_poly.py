"""Fits the cubic used by the prefill kernel to evaluate 2^f on the FMA pipe, f in [-1/2, 1/2].

2^x is split as 2^n * 2^f with n = round(x) and f = x - n (Cody-Waite style range reduction; n comes from the
1.5 * 2^23 rounding trick, and 2^n is applied by adding n to the exponent bits). The cubic minimises the maximum
relative error on [-1/2, 1/2] (Remez exchange on the relative error, double precision). Its error, about 1e-4,
is far below the bf16 rounding (2^-9) that every probability goes through next.

Run: python head_sparse_paged_b200/csrc/fit_exp2_poly.py  -> prints the coefficients pasted into prefill_sm100.cuh.
"""
import numpy as np


def remez_rel(fn, lo, hi, deg, iters=30):
    k = np.arange(deg + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))     # Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    c = None
    for _ in range(iters):
        # solve sum c_i x^i - (-1)^k E f(x) = f(x) for c and E (relative error levels)
        A = np.zeros((deg + 2, deg + 2))
        for i in range(deg + 1):
            A[:, i] = x ** i
        A[:, deg + 1] = ((-1.0) ** k) * fn(x)
        sol = np.linalg.solve(A, fn(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - fn(grid)) / fn(grid)
        # new reference: extrema of err in each sign-alternating segment
        idx = [0]
        for j in range(1, len(grid) - 1):
            if (err[j] - err[j - 1]) * (err[j + 1] - err[j]) <= 0:
                idx.append(j)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        ecand = err[idx]
        # keep deg+2 alternating points with the largest magnitudes
        pts = [(cand[0], ecand[0])]
        for xx, ee in zip(cand[1:], ecand[1:]):
            if np.sign(ee) == np.sign(pts[-1][1]):
                if abs(ee) > abs(pts[-1][1]):
                    pts[-1] = (xx, ee)
            else:
                pts.append((xx, ee))
        while len(pts) > deg + 2:
            if abs(pts[0][1]) < abs(pts[-1][1]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) == deg + 2:
            x = np.array([p[0] for p in pts])
    err = (np.polyval(c[::-1], grid) - fn(grid)) / fn(grid)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_rel(lambda t: np.exp2(t), -0.5, 0.5, 3)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    p = np.float32(c32[3])
    for ci in c32[2::-1]:
        p = (p * f + ci).astype(np.float32)
    e32 = float(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max())
    print("coefficients c0..c3 (float32):", [float(v).hex() for v in c32], [repr(float(v)) for v in c32])
    print(f"max relative error: {e:.3e} (double), {e32:.3e} (float32 Horner)")
