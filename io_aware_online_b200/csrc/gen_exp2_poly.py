"""Fit the polynomial the prefill kernel uses to evaluate part of its exp2 work on
the FMA pipe instead of the MUFU unit.

Method: 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f is
approximated by a polynomial P(f) = c0 + c1 f + ... + cn f^n whose maximum
RELATIVE error on [-1/2, 1/2] is minimised by the Remez exchange algorithm
(equioscillation of the weighted error e(f) = (P(f) - 2^f) / 2^f at n + 2
points).  2^j is then applied by adding j to the exponent field of P(f).

Run: python io_aware_online_b200/csrc/gen_exp2_poly.py [degree]
Prints the coefficients c0..cn and the achieved max relative error.
"""
import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 30):
    a, b = -0.5, 0.5
    # unknowns: c0..c_deg and the levelled error E
    n = deg + 2                                   # number of reference points
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        rhs = np.zeros(n)
        for i, xi in enumerate(x):
            t = 2.0 ** xi
            for k in range(deg + 1):
                A[i, k] = xi ** k / t        # (P(x_i) - 2^x_i) / 2^x_i = (-1)^i E
            A[i, deg + 1] = -((-1.0) ** i)
            rhs[i] = 1.0
        sol = np.linalg.solve(A, rhs)
        c = sol[:deg + 1]
        # new reference: extrema of the relative error on a fine grid
        g = np.linspace(a, b, 200001)
        p = sum(c[k] * g ** k for k in range(deg + 1))
        err = (p - 2.0 ** g) / 2.0 ** g
        # split the grid into n sign-alternating segments and take each segment's extremum
        idx = [0]
        for i in range(1, len(g)):
            if np.sign(err[i]) != np.sign(err[idx[-1]]) and err[i] != 0:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep the n largest alternating extrema (contiguous window with the max)
        best = max(range(len(idx) - n + 1), key=lambda s: min(abs(err[idx[s + j]]) for j in range(n)))
        x = g[idx[best:best + n]]
    g = np.linspace(a, b, 400001)
    p = sum(c[k] * g ** k for k in range(deg + 1))
    return c, float(np.max(np.abs((p - 2.0 ** g) / 2.0 ** g)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    for k, v in enumerate(c):
        print(f"c{k} = {np.float32(v)!r}  ({v:.12e})")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
