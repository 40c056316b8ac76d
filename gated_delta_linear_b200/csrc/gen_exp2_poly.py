"""Fit the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the FMA-pipe exp2.

Method: Remez exchange for the minimax *relative* error of a degree-3
polynomial (E. Remez, 1934), started from Chebyshev nodes.  The kernel uses it
after Cody-Waite range reduction (W. J. Cody and W. Waite, "Software Manual for
the Elementary Functions", 1980): x = n + f with n = round(x), so
2^x = 2^n * p(f), where 2^n is added to the exponent field.

Run: python gated_delta_linear_b200/csrc/gen_exp2_poly.py
Prints the coefficients (c0..c3, ascending) and the max relative error.
"""

import numpy as np

DEG = 3
A, B = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (A + B) + 0.5 * (B - A) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    for _ in range(iters):
        f = np.exp2(x)
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)  (relative-error equioscillation)
        M = np.zeros((n, n))
        for j in range(deg + 1):
            M[:, j] = x ** j
        M[:, deg + 1] = (-1.0) ** k * f
        sol = np.linalg.solve(M, f)
        c = sol[: deg + 1]
        # new extrema of the relative error
        g = np.linspace(A, B, 200001)
        e = (np.polyval(c[::-1], g) - np.exp2(g)) / np.exp2(g)
        idx = [0]
        for i in range(1, len(g) - 1):
            if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
                idx.append(i)
        idx.append(len(g) - 1)
        idx = np.array(idx)
        if len(idx) >= n:
            # keep the n extrema with alternating signs and largest magnitude
            best = sorted(idx, key=lambda i: -abs(e[i]))[:n]
            x = np.sort(g[best])
    g = np.linspace(A, B, 400001)
    err = np.max(np.abs((np.polyval(c[::-1], g) - np.exp2(g)) / np.exp2(g)))
    return c, err


if __name__ == "__main__":
    c, err = remez()
    c32 = c.astype(np.float32)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}f  ({ci.view(np.uint32):#010x})")
    print(f"max relative error (float64 evaluation): {err:.3e}")
