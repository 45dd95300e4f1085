"""Derives the coefficients of the software 2^f used by the attention
softmax for part of its exponentials (the rest go to the MUFU ex2 unit).

Method (published, textbook): Cody-Waite range reduction x = j + f with
j = round-to-nearest(x) and f in [-1/2, 1/2], then 2^x = 2^j * p(f) where p
is the degree-3 polynomial of minimax *relative* error to 2^f on
[-1/2, 1/2], found with the Remez exchange algorithm (equioscillation of the
weighted error at deg + 2 points).  2^j is applied by adding j to the
exponent field.

Run:  python exp2_poly_fit.py   -> prints the float32 coefficients and the
bound; the kernel header holds the printed values.
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)  # noqa: E731
    n = deg + 2
    # initial reference: Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve sum_k c_k x_i^k + (-1)^i E f(x_i) = f(x_i)  (relative weighting)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(xi)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between its sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        ecand = err[idx]
        # keep n alternating extrema of largest magnitude
        sel = [0]
        for i in range(1, len(cand)):
            if np.sign(ecand[i]) == np.sign(ecand[sel[-1]]):
                if abs(ecand[i]) > abs(ecand[sel[-1]]):
                    sel[-1] = i
            else:
                sel.append(i)
        while len(sel) > n:
            sel.pop(0 if abs(ecand[sel[0]]) < abs(ecand[sel[-1]]) else -1)
        if len(sel) == n:
            x = cand[sel]
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001)
    e32 = np.abs((np.polyval(c32[::-1].astype(np.float64), g) - np.exp2(g)) / np.exp2(g)).max()
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32)")
