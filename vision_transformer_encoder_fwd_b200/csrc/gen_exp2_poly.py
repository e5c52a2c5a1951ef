"""Fit the polynomial the attention kernel uses for 2^f on f in [-1/2, 1/2].

The attention softmax splits exp2(x) = 2^j * 2^f with j = round(x) and f = x - j (Cody-Waite
range reduction; the rounding is done by adding 1.5 * 2^23, so it stays on the FMA pipe) and
evaluates 2^f with a cubic on the FMA pipe for part of the elements, relieving the special
function unit.  This script derives the cubic p(f) = c0 + c1 f + c2 f^2 + c3 f^3 by a Remez
exchange that minimises the maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2].  Run it to
reproduce the coefficients written in attention.cuh:

    python vision_transformer_encoder_fwd_b200/csrc/gen_exp2_poly.py
"""
import numpy as np


def fit(degree=3, iters=50, lo=-0.5, hi=0.5):
    n = degree + 1                                     # unknowns c0..c_degree, plus the level E
    x = lo + (hi - lo) * (0.5 - 0.5 * np.cos(np.linspace(0, np.pi, n + 1)))
    grid = np.linspace(lo, hi, 400001)
    for _ in range(iters):
        A = np.zeros((n + 1, n + 1))
        for i, xi in enumerate(x):
            A[i, :n] = [xi ** k / 2.0 ** xi for k in range(n)]
            A[i, n] = (-1) ** i
        c = np.linalg.solve(A, np.ones(n + 1))[:n]
        err = sum(c[k] * grid ** k for k in range(n)) / 2.0 ** grid - 1
        # new reference set: one extremum per sign run of the error, the n+1 largest in a row
        runs, start = [], 0
        sg = np.sign(err)
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sg[i] != sg[start]:
                j = start + int(np.argmax(np.abs(err[start:i])))
                runs.append(j)
                start = i
        if len(runs) < n + 1:
            break
        best = max(range(len(runs) - n), key=lambda s: min(abs(err[runs[s + t]]) for t in range(n + 1)))
        x = grid[runs[best:best + n + 1]]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = fit()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print("max relative error on [-1/2, 1/2]: %.3e" % e)
    print("as float32:", ", ".join(repr(float(np.float32(v))) for v in c))
