"""Fits the polynomial the prefill kernel uses to evaluate 2^f on the FMA pipe.

    python attn_fwd_05_b200/csrc/fit_exp2_poly.py

Method (Cody and Waite's range reduction, then a minimax fit): the kernel splits
x = n + f with n = round-to-nearest(x) and f in [-1/2, 1/2], evaluates 2^f with a
degree-3 polynomial in Horner form and adds n to the exponent field of the result.
This script finds the degree-3 polynomial that minimises the maximum *relative* error
of 2^f on [-1/2, 1/2] by the Remez exchange algorithm (Chebyshev nodes as the start,
then alternate between solving the levelled-error linear system and moving each
reference point to a local extremum of the error), rounds the coefficients to fp32
and prints them with the achieved error.  The kernel's probabilities are rounded to
bf16 (relative step 2^-8), so an error around 1e-4 is far below what the output keeps.
"""

from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg: int = DEG, iters: int = 30):
    m = deg + 2
    k = np.arange(m)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (m - 1 - k) / (m - 1))  # Chebyshev extrema
    grid = np.linspace(LO, HI, 200001)
    target = np.exp2(grid)
    coef = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  (levelled relative error)
        A = np.zeros((m, m))
        for j in range(deg + 1):
            A[:, j] = x ** j
        A[:, deg + 1] = -((-1.0) ** k) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        coef = sol[: deg + 1]
        err = (np.polyval(coef[::-1], grid) - target) / target
        # new reference: one extremum of the error in each sign-alternating segment
        s = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < m:
            break
        idx = np.array(idx)
        while len(idx) > m:  # drop the smallest end
            idx = idx[1:] if abs(err[idx[0]]) < abs(err[idx[-1]]) else idx[:-1]
        x = grid[idx]
    return coef


def main():
    coef = remez()
    c32 = coef.astype(np.float32)
    grid = np.linspace(LO, HI, 400001)
    approx = np.polyval(c32.astype(np.float64)[::-1], grid)
    rel = np.abs(approx / np.exp2(grid) - 1).max()
    for i, c in enumerate(c32):
        print(f"c{i} = {float(c).hex()}  ({float(c):.9g})")
    print(f"max relative error on [{LO}, {HI}]: {rel:.3e}")


if __name__ == "__main__":
    main()
