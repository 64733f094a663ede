"""Fits the polynomial behind the FMA-pipe exp2 of the attention kernel.

    python context_attention_dits_cp_b200/csrc/fit_exp2_poly.py [degree]

The kernel computes 2^x for a fraction of the softmax elements on the FMA
pipe instead of the MUFU unit (which the softmax otherwise saturates):
Cody-Waite style range reduction x = n + f with n = round(x), f in
[-1/2, 1/2]; 2^f from a polynomial p(f); 2^n by adding n to the float's
exponent field.  This script finds p as the minimax approximation of 2^f in
RELATIVE error on [-1/2, 1/2] with the Remez exchange algorithm (float64),
then rounds the coefficients to float32 and reports the relative error the
float32 polynomial actually reaches.  The printed constants are the ones
compiled into attn_tc.cu.
"""
from __future__ import annotations

import sys

import numpy as np

LO, HI = -0.5, 0.5


def remez_relative(deg: int, iters: int = 40):
    f = lambda x: np.exp2(x)
    w = lambda x: 1.0 / np.exp2(x)           # relative error weight
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (n - 1))   # Chebyshev nodes
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E / w(x_i) = f(x_i) for coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i / w(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) * w(grid)
        # new reference: the extrema of the error between its sign changes
        sign = np.sign(err)
        idx = [0]
        for j in range(1, len(grid)):
            if sign[j] != sign[idx[-1]]:
                idx.append(j)
            elif abs(err[j]) > abs(err[idx[-1]]):
                idx[-1] = j
        if len(idx) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best, best_i = -1.0, 0
        for s in range(len(idx) - n + 1):
            m = min(abs(err[idx[s:s + n]]))
            if m > best:
                best, best_i = m, s
        x = grid[idx[best_i:best_i + n]]
    return c


def fp32_relative_error(c32):
    g = np.linspace(LO, HI, 400001).astype(np.float32)
    p = np.float32(c32[-1])
    for ck in c32[-2::-1]:
        p = np.float32(p * g + np.float32(ck))    # Horner in float32, one rounding per step
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(g.astype(np.float64)) - 1.0)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c = remez_relative(deg)
    c32 = [np.float32(v) for v in c]
    print(f"degree {deg} minimax of 2^f on [{LO}, {HI}] (relative error)")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v):.9e}f   // 0x{np.float32(v).view(np.uint32):08x}")
    print(f"  max relative error with float32 coefficients: {fp32_relative_error(c32):.3e}")


if __name__ == "__main__":
    main()
