"""Derive the coefficients of the polynomial 2^f used by the kernels'
FMA-pipe exponential, and print them as a C++ table.

Method: Remez exchange for the minimax *relative* error of a degree-d
polynomial p(f) ~ 2^f on f in [-1/2, 1/2] (Remez, 1934; the weighted form as
in Cheney, "Introduction to Approximation Theory", ch. 3).  The kernels reduce
x = n + f with n = rint(x) and form 2^x = p(f) * 2^n by adding n to the
exponent field, so only [-1/2, 1/2] is needed.

    python gen_exp2_poly.py [degree]      # default 5 (the degree the kernels use)
"""
import sys

import numpy as np


def remez_exp2(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 60):
    """Minimax coefficients (c0..cdeg) of 2^f on [a, b] in relative error, and that error."""
    n = deg + 2  # reference points
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    c = None
    E = 0.0
    for _ in range(iters):
        # solve p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i}  for c and E (relative error weight)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        rhs = 2.0 ** x
        sol = np.linalg.solve(A, rhs)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of err with alternating signs, one per sign run
        s = np.sign(err)
        s[s == 0] = 1
        idx = []
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or s[i] != s[start]:
                seg = slice(start, i)
                j = start + int(np.argmax(np.abs(err[seg])))
                idx.append(j)
                start = i
        if len(idx) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = None
        for off in range(len(idx) - n + 1):
            cand = idx[off:off + n]
            m = np.min(np.abs(err[cand]))
            if best is None or m > best[0]:
                best = (m, cand)
        xn = grid[best[1]]
        if np.allclose(xn, x, atol=1e-12):
            break
        x = xn
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.max(np.abs(err)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c, e = remez_exp2(deg)
    print(f"// degree {deg} minimax (relative) fit of 2^f on [-1/2, 1/2]; max rel. error {e:.3e}")
    print("#define LARD_EXP2_POLY {%s}" % ", ".join("%.9ef" % v for v in c))


if __name__ == "__main__":
    main()
