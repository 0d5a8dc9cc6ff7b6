"""Derives the polynomial used by the forward kernel's FMA-pipe exp2.

2^x is split Cody-Waite style as x = n + f with n = round(x) and
f in [-1/2, 1/2]; then 2^x = 2^n * 2^f, where 2^n is an exponent-field add
and 2^f is approximated by a cubic.  The cubic minimises the maximum
*relative* error on [-1/2, 1/2] (Remez exchange on the error
w(f) * (p(f) - 2^f) with weight w = 2^-f), computed here in float64 and
rounded to float32.

    python sparse_attention_attn_b200/csrc/derive_exp2_poly.py

prints the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the relative error
bound of the float32 coefficients, measured on a dense grid.
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg: int = DEG, iters: int = 40):
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E * 2^x_i  (relative error alternation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(sorted(set(idx)))
        # keep the n points with largest |err| that alternate in sign
        cand = idx[np.argsort(-np.abs(err[idx]))]
        chosen = []
        for i in sorted(cand[: max(n * 4, n)]):
            chosen.append(i)
        chosen = sorted(chosen)
        # enforce alternation greedily
        alt = [chosen[0]]
        for i in chosen[1:]:
            if np.sign(err[i]) == np.sign(err[alt[-1]]):
                if abs(err[i]) > abs(err[alt[-1]]):
                    alt[-1] = i
            else:
                alt.append(i)
        if len(alt) < n:
            break
        # take the n consecutive points with the largest minimum |err|
        best, best_j = -1.0, 0
        for j in range(len(alt) - n + 1):
            m = np.min(np.abs(err[alt[j:j + n]]))
            if m > best:
                best, best_j = m, j
        x = grid[alt[best_j:best_j + n]]
    return c


def max_rel_err_f32(c) -> float:
    c32 = np.asarray(c, dtype=np.float32)
    f = np.linspace(LO, HI, 400001).astype(np.float32)
    p = np.zeros_like(f)
    for ci in c32[::-1]:  # Horner in float32, as the kernel evaluates it
        p = (p * f + ci).astype(np.float32)
    ref = 2.0 ** f.astype(np.float64)
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    c = remez()
    c32 = np.asarray(c, dtype=np.float32)
    print("coefficients (c0..c3, float32):")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci):.9e}f  (hex {np.float32(ci).view(np.uint32):#010x})")
    print(f"max relative error on [-1/2, 1/2] (float32 Horner): {max_rel_err_f32(c32):.3e}")
