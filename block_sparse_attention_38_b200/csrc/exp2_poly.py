"""Coefficients of the polynomial 2^f the forward kernel evaluates on the FMA pipe.

    python block_sparse_attention_38_b200/csrc/exp2_poly.py

Method (Cody and Waite's range reduction, then a minimax fit): for
x = n + f with n = rint(x) and f in [-1/2, 1/2], 2^x = 2^n * 2^f; 2^f is
approximated by the degree-3 polynomial c0 + c1 f + c2 f^2 + c3 f^3 whose
maximum *relative* error over [-1/2, 1/2] is smallest, found by Remez
exchange (equioscillation of the weighted error at 5 points).  Evaluated in
fp32 with fused multiply-adds the result is within 1e-4 relative of 2^x,
well below the bf16 rounding (2^-9) that P receives.  The script prints the
coefficients as fp32 literals and the fp32-evaluated error bound.
"""
import numpy as np


def remez(deg=3, lo=-0.5, hi=0.5, iters=30):
    k = np.arange(deg + 2)
    xs = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k[::-1] / (deg + 1))  # Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve sum c_i x^i - 2^x = (-1)^j E 2^x at the reference points
        A = np.zeros((deg + 2, deg + 2))
        for j, x in enumerate(xs):
            A[j, :deg + 1] = x ** np.arange(deg + 1)
            A[j, deg + 1] = (-1) ** j * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep deg + 2 alternating points of largest |err|
        pts = sorted(idx, key=lambda i: -abs(err[i]))[:deg + 2]
        xs = np.sort(grid[pts])
    return c, np.abs(err).max()


def fp32_error(c):
    c32 = np.float32(c)
    x = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    p = np.full_like(x, c32[3])
    for k in (2, 1, 0):
        p = (p * x + c32[k]).astype(np.float32)
    return np.abs(p.astype(np.float64) / 2.0 ** x.astype(np.float64) - 1.0).max()


if __name__ == "__main__":
    c, e = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {float(np.float32(v)):.9g}f  ({v:.17g})")
    print(f"max relative error: minimax {e:.3e}, fp32 evaluation {fp32_error(c):.3e}")
