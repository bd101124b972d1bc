"""Minimax polynomial for 2^f on [-1/2, 1/2] (relative error), by Remez exchange.

The flash kernels evaluate part of their exponentials on the FMA pipe instead
of the MUFU unit (`exp2_poly2` in tc_ptx.cuh): y = j + f with j = rint(y) and
|f| <= 1/2, 2^f from a degree-3 polynomial, 2^j added to the exponent field.
This script derives that polynomial's coefficients and its error bound; the
constants in tc_ptx.cuh are its output rounded to float32, and
tests/test_exp2_poly.py checks the two against each other.

    python exp2_poly.py        # prints the coefficients and max relative error
"""
import numpy as np


def minimax_exp2(n, a=-0.5, b=0.5, iters=40, grid=200001):
    """Coefficients c[0..n] (ascending powers) minimising max |p(f)/2^f - 1| on [a, b].

    Remez exchange for a weighted (relative) error: solve
    p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i} on n+2 reference points, then move the
    references to the alternating extrema of the error on a fine grid.
    """
    k = np.arange(n + 2)
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))  # Chebyshev start
    g = np.linspace(a, b, grid)
    c = None
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n + 1]
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
        # interior extrema (sign changes of the slope) plus both end points
        s = np.sign(np.diff(err))
        ext = np.concatenate(([0], np.nonzero(s[1:] != s[:-1])[0] + 1, [grid - 1]))
        if len(ext) < n + 2:
            break
        # keep, among runs of equal error sign, the largest |err|; then the n+2 largest
        keep = []
        for i in ext:
            if keep and np.sign(err[i]) == np.sign(err[keep[-1]]):
                if abs(err[i]) > abs(err[keep[-1]]):
                    keep[-1] = i
            else:
                keep.append(i)
        while len(keep) > n + 2:  # drop the smaller end
            keep.pop(0 if abs(err[keep[0]]) < abs(err[keep[-1]]) else -1)
        if len(keep) < n + 2:
            break
        x = g[np.array(keep)]
    err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    for n in (3, 4):
        c, e = minimax_exp2(n)
        print(f"degree {n}: coefficients (float32, ascending) "
              f"{[float(np.float32(v)) for v in c]}  max relative error {e:.3e}")
