"""Fit the polynomial the prefill softmax uses to evaluate 2^f on f in [-1/2, 1/2] on the FMA pipe.

Method: Remez exchange (E. Ya. Remez, 1934) for the minimax *relative* error of a degree-n
polynomial P(f) ~ 2^f, solved in float64 on a dense grid; the coefficients are then rounded to
float32 and the achieved error is re-measured with the rounded coefficients.  The kernel splits
x = n + f (n = nearest integer, obtained with the 1.5 * 2^23 round-to-integer addition), evaluates
P(f) by Horner's rule and adds n to the exponent field.

    python fit_exp2_poly.py [degree]      # prints the coefficients and the error bound
"""
import sys

import numpy as np


def remez_exp2(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 40):
    f = lambda x: np.exp2(x)
    # Chebyshev extrema as the initial reference
    k = np.arange(deg + 2)
    ref = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (deg + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve P(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of the error
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < deg + 2:
            break
        # keep deg+2 consecutive extrema with the largest minimum
        best = max(range(len(idx) - deg - 1), key=lambda s: min(abs(err[idx[s:s + deg + 2]])))
        ref = grid[idx[best:best + deg + 2]]
    return c


def measured_error(c32):
    x = np.linspace(-0.5, 0.5, 2000001)
    p = np.zeros_like(x, dtype=np.float32)
    xs = x.astype(np.float32)
    for ci in c32[::-1]:
        p = (p * xs + ci).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) - np.exp2(xs.astype(np.float64))) / np.exp2(xs.astype(np.float64))))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez_exp2(deg)
    c32 = np.array(c, dtype=np.float32)
    print(f"degree {deg}: max relative error {measured_error(c32):.3e} (float32 coefficients, Horner)")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci)!r}f  ({float(ci).hex()})")
