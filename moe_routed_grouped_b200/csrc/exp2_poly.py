"""Coefficients of the polynomial used for 2^f, f in [-1/2, 1/2], in the
attention kernel's software exponential.

The kernel splits y = j + f with j = rint(y) (float32 add/subtract of
1.5 * 2^23), evaluates p(f) ~ 2^f with Horner's rule, and forms 2^y by adding
j to the exponent field of p(f).  p minimises the maximum RELATIVE error
|p(f) / 2^f - 1| over the interval (Remez exchange on a dense grid), which is
what matters for the fp16-rounded probabilities it feeds.

Run: python exp2_poly.py [degree]    (prints coefficients and the error)
"""
import sys

import numpy as np


def remez_relative(deg: int, lo=-0.5, hi=0.5, iters=40, grid=20001):
    x = np.linspace(lo, hi, grid)
    f = np.exp2(x)
    # start from Chebyshev extrema
    n = deg + 2
    ref = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    coef = None
    for _ in range(iters):
        # solve p(x_i)/f(x_i) - 1 = (-1)^i E  for coefficients and E
        A = np.zeros((n, n))
        for i, xi in enumerate(ref):
            A[i, :deg + 1] = xi ** np.arange(deg + 1) / np.exp2(xi)
            A[i, deg + 1] = (-1) ** i
        sol = np.linalg.solve(A, np.ones(n))
        coef = sol[:deg + 1]
        err = np.polyval(coef[::-1], x) / f - 1.0
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, grid - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid - 1)
        idx = np.array(idx)
        if len(idx) >= n:
            # keep the n largest alternating extrema
            cand = idx[np.argsort(-np.abs(err[idx]))][:n]
            ref = np.sort(x[cand])
    err = np.polyval(coef[::-1], x) / f - 1.0
    return coef, float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_relative(deg)
    c32 = c.astype(np.float32)
    x = np.linspace(-0.5, 0.5, 200001)
    p32 = np.zeros_like(x, dtype=np.float32)
    for ci in c32[::-1]:
        p32 = p32 * x.astype(np.float32) + ci
    e32 = float(np.max(np.abs(p32.astype(np.float64) / np.exp2(x) - 1.0)))
    print(f"degree {deg}: max relative error {e:.3e} (float32 Horner {e32:.3e})")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci):.9e}f")
