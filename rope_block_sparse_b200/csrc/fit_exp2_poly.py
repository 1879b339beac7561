"""Fit the polynomial behind the FMA-pipe exp2 of the attention softmax.

Remez exchange for the polynomial of a given degree minimising the maximum
RELATIVE error of 2^f on [-1/2, 1/2]; prints the max error and the float32
coefficients c0..cn (2^f ~ c0 + c1 f + ... + cn f^n).  The degree-3 result is
the one compiled into attention.cu:
    python rope_block_sparse_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def remez(deg, a=-0.5, b=0.5, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    t = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])  # relative-error weight
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], t) - np.exp2(t)) / np.exp2(t)
        d = np.diff(err)
        ext = np.where(np.sign(d[1:]) != np.sign(d[:-1]))[0] + 1
        pts = np.concatenate(([0], ext, [len(t) - 1]))
        if len(pts) != n:
            pts = np.sort(pts[np.argsort(-np.abs(err[pts]))[:n]])
        x = t[pts]
    c32 = c.astype(np.float32)
    err32 = (np.polyval(c32.astype(np.float64)[::-1], t) - np.exp2(t)) / np.exp2(t)
    return c32, float(np.max(np.abs(err32)))


if __name__ == "__main__":
    for deg in (2, 3, 4):
        c, e = remez(deg)
        print(f"degree {deg}: max relative error {e:.3e}; coefficients {[float(v) for v in c]}")
