"""Fits the polynomial the forward kernel uses to evaluate 2^f on the FMA pipe.

Method: Cody-Waite style range reduction x = j + f with j = round(x), f in [-1/2, 1/2]
(2^x = 2^j * 2^f, the 2^j factor applied by adding j to the exponent bits), and a
minimax polynomial p(f) ~ 2^f in the relative-error sense, found with the Remez exchange
algorithm (E. Remez, 1934): solve for the coefficients that equioscillate on n+2
reference points, move the points to the extrema of the error, repeat.

    python attention_kl_divergence_02_b200/csrc/fit_exp2_poly.py [degree]

prints the coefficients (c0 .. cn) as fp32 literals and the worst relative error of the
fp32 Horner evaluation over a dense grid.
"""
import sys

import numpy as np


def remez_exp2(n, iters=30):
    lo, hi = -0.5, 0.5
    k = np.arange(n + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n + 1 - k) / (n + 1))  # Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}   (equioscillating relative error)
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, :n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum of the error per sign-alternating segment
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        idx = np.array(idx)
        if len(idx) > n + 2:  # keep the n+2 consecutive extrema with the largest minimum
            best = max(range(len(idx) - n - 1), key=lambda s: np.min(np.abs(err[idx[s:s + n + 2]])))
            idx = idx[best:best + n + 2]
        if len(idx) == n + 2:
            x = grid[idx]
    return c


def fp32_horner(c, f):
    c32 = [np.float32(v) for v in c]
    f = f.astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for v in reversed(c32[:-1]):
        acc = (acc * f + v).astype(np.float32)   # fma rounds once; this rounds twice (worse)
    return acc


def main():
    n = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = remez_exp2(n)
    f = np.linspace(-0.5, 0.5, 2000001)
    rel = np.abs(fp32_horner(c, f).astype(np.float64) / 2.0 ** f - 1.0)
    print("degree %d, max relative error %.3e (fp32 Horner)" % (n, rel.max()))
    for i, v in enumerate(c):
        print("c%d = %.9ef" % (i, np.float32(v)))


if __name__ == "__main__":
    main()
