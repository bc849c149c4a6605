"""Fit the polynomial behind exp2_poly2() in fa_ptx.cuh.

2^x is evaluated on the FMA pipe by Cody-Waite range reduction: x = n + f
with n = round(x) and f in [-1/2, 1/2], then 2^x = 2^n * p(f).  p is the
degree-3 minimax approximation of 2^f on [-1/2, 1/2] in relative error,
found here with the Remez exchange algorithm.  Run:

    python io_aware_exact_forward_b200/csrc/fit_exp2_poly.py

and it prints the float32 coefficients (c0..c3) and the float32 Horner error.
"""

import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        cand = [0] + [i for i in range(1, len(grid) - 1)
                      if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(grid) - 1]
        pts = []
        for i in sorted(cand):
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        if len(pts) >= n:
            k = max(range(len(pts) - n + 1), key=lambda s: min(abs(err[pts[s:s + n]])))
            x = grid[pts[k:k + n]]
    return c


def main():
    c = remez(3).astype(np.float32)
    t = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    p = np.float32(c[3])
    for k in (2, 1, 0):
        p = (p * t + c[k]).astype(np.float32)
    ref = np.exp2(t.astype(np.float64))
    rel = np.max(np.abs(p.astype(np.float64) - ref) / ref)
    print("c0..c3 =", [float(v) for v in c])
    print("max relative error (float32 Horner on [-1/2, 1/2]) = %.3e" % rel)


if __name__ == "__main__":
    main()
