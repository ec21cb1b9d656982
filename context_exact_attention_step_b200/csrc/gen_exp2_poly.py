"""Coefficients of the polynomial 2^f ~ p(f) on f in [-1/2, 1/2] used by the
softmax kernel's software exp2.

Method: Cody and Waite style range reduction, 2^x = 2^n * 2^f with
n = round(x) and f = x - n in [-1/2, 1/2], followed by a minimax polynomial
for 2^f in the relative-error sense.  The minimax fit is computed here with
the Remez exchange algorithm on a dense grid (a textbook method, no library
routine is copied).  Run it to print the coefficients and their error bound:

    python gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_exp2(degree, iters=30, grid=200001):
    """Minimax (relative error) polynomial for 2^f on [-1/2, 1/2]."""
    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    n = degree + 2
    # Chebyshev extrema as the initial reference set
    k = np.arange(n)
    ref = 0.5 * np.cos(np.pi * k / (n - 1))[::-1]
    for _ in range(iters):
        # solve p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i} for coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(ref))
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], f) - target) / target
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, grid - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(grid - 1)
        idx = np.array(sorted(set(idx)))
        # keep the n largest alternating extrema
        cand = idx[np.argsort(-np.abs(err[idx]))]
        chosen = []
        for i in cand:
            if all(abs(i - j) > grid // (8 * n) for j in chosen):
                chosen.append(i)
            if len(chosen) == n:
                break
        ref = np.sort(f[np.array(chosen)])
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    # evaluate the float32 Horner form as the kernel does
    f32 = np.float32
    cs = [f32(x) for x in c]
    x = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    p = np.zeros_like(x) + cs[-1]
    for coef in cs[-2::-1]:
        p = p * x + coef
    e32 = float(np.max(np.abs(p.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)))
    print(f"degree {deg}: minimax relative error {e:.3e} (float32 Horner {e32:.3e})")
    for i, v in enumerate(cs):
        print(f"  c{i} = {float(v):.9e}f")
