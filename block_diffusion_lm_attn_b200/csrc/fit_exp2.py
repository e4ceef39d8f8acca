"""Fits the polynomial the attention kernels use to evaluate 2^f on the FMA
pipes for part of the softmax (the rest goes to the special-function unit).

Method: Cody-Waite style range reduction, 2^x = 2^n * 2^f with n = round(x)
and f = x - n in [-1/2, 1/2], then 2^f from a degree-3 polynomial whose
coefficients minimise the maximum RELATIVE error on [-1/2, 1/2].  The
minimax fit is computed here with the Remez exchange algorithm (Remez 1934),
starting from a least-squares fit on Chebyshev nodes, all in float64; the
coefficients are then rounded to float32 and the error of the rounded
polynomial is reported.

Run:  python fit_exp2.py      (prints the coefficients and the error bound)
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def rel_err(c, x):
    return np.polyval(c[::-1], x) / np.exp2(x) - 1.0


def remez(deg=DEG, iters=30):
    n = deg + 2
    # initial reference: Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    c = None
    for _ in range(iters):
        # solve sum_j c_j x_i^j - (-1)^i E 2^x_i = 2^x_i  (relative error)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        # new reference: extrema of the error on a fine grid
        g = np.linspace(LO, HI, 200001)
        e = rel_err(c, g)
        idx = [0]
        for i in range(1, len(g) - 1):
            if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
                idx.append(i)
        idx.append(len(g) - 1)
        cand = g[idx]
        ecand = np.abs(e[idx])
        if len(cand) >= n:
            # keep n alternating points with the largest errors
            order = np.argsort(-ecand)[:n]
            x = np.sort(cand[order])
    return c


def main():
    c = remez()
    c32 = c.astype(np.float32).astype(np.float64)
    g = np.linspace(LO, HI, 1000001)
    print("degree %d minimax coefficients (c0..c%d), float32:" % (DEG, DEG))
    for i, v in enumerate(c.astype(np.float32)):
        print("  c%d = %.9e  (0x%08x)" % (i, v, np.float32(v).view(np.uint32)))
    print("max relative error (float64 eval of float32 coefficients): %.3e"
          % np.abs(rel_err(c32, g)).max())


if __name__ == "__main__":
    main()
