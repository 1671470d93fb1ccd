"""Coefficients of the polynomial exp2 used by the softmax kernels.

Cody & Waite style range reduction (x = j + f, j = round(x), f in
[-0.5, 0.5]) followed by a degree-3 minimax polynomial p(f) ~ 2^f in
relative error, fitted here with the Remez exchange algorithm; 2^x is then
assembled by adding j to the exponent field of p(f).  Prints the fp32
coefficients and the maximum relative error (about 7.5e-5, far below the
2^-9 rounding of the bf16 probabilities that consume it).

    python fit_exp2_poly.py
"""
import numpy as np


def remez(deg=3, a=-0.5, b=0.5, iters=40):
    n = deg + 2
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))
    g = np.linspace(a, b, 400001)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        y = 2.0 ** x
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * y[i]
        c = np.linalg.solve(A, y)[:deg + 1]
        err = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        idx = [0] + [k for k in range(1, len(g) - 1)
                     if (err[k] - err[k - 1]) * (err[k + 1] - err[k]) < 0] + [len(g) - 1]
        if len(idx) != n:
            break
        x = g[idx]
    c32 = c.astype(np.float32)
    err32 = (np.polyval(c32[::-1].astype(np.float64), g) - 2.0 ** g) / 2.0 ** g
    return c32, float(np.max(np.abs(err32)))


if __name__ == "__main__":
    c, e = remez()
    print("coefficients c0..c3:", ", ".join("%.9ef" % v for v in c))
    print("max relative error: %.3e" % e)
