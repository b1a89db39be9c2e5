#!/usr/bin/env python3
"""Fits the polynomial the attention kernel uses to evaluate 2^f, f in [0, 1),
on the FMA pipe (a share of the softmax exponentials is computed this way
instead of on the special-function unit).

Method: minimax (Chebyshev) approximation of 2^f on [0, 1) in the relative
error, by the Remez exchange algorithm (Remez 1934; e.g. Muller, "Elementary
Functions", ch. 3), with the constraint p(0) = 1 so that 2^j * p(0) is exact
and the exponential is exactly 1 at the running maximum.  Form:

    p(f) = 1 + f * (a1 + f * (a2 + f * a3))

Relative error e(f) = (p(f) - 2^f) / 2^f.  With three free coefficients the
equioscillation has four alternation points in (0, 1].

Prints the coefficients as float32 literals together with the relative error
of the fp32 Horner evaluation on a dense grid.  The kernel's exponentials feed
bf16 probabilities (relative spacing 2^-8), so a relative error around 1e-4
is invisible in P and adds at most that much to the softmax normaliser.
"""
from __future__ import annotations

import numpy as np


def fit(degree: int = 3, iters: int = 30):
    n = degree  # free coefficients a1..a_degree
    # initial reference: Chebyshev-like points in (0, 1]
    k = np.arange(n + 1)
    x = 0.5 - 0.5 * np.cos(np.pi * (k + 0.5) / (n + 1))
    x[-1] = 1.0
    grid = np.linspace(0.0, 1.0, 200001)[1:]
    a = None
    for _ in range(iters):
        # solve  sum_i a_i x^i - 2^x = (-1)^k E 2^x  for a_1..a_n, E  (p(0) = 1 fixed)
        A = np.zeros((n + 1, n + 1))
        rhs = np.zeros(n + 1)
        for r, xr in enumerate(x):
            w = 2.0 ** xr
            for i in range(1, n + 1):
                A[r, i - 1] = xr ** i
            A[r, n] = -((-1) ** r) * w
            rhs[r] = w - 1.0
        sol = np.linalg.solve(A, rhs)
        a = sol[:n]
        err = rel_err(a, grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(s))[0] + 1, [len(grid)]))
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(idx[:-1], idx[1:])]
        if len(ext) >= n + 1:
            ext = sorted(ext, key=lambda i: -abs(err[i]))[: n + 1]
            x = np.sort(grid[ext])
    return a


def rel_err(a, f):
    p = np.ones_like(f)
    acc = np.zeros_like(f)
    for c in a[::-1]:
        acc = acc * f + c
    p = 1.0 + f * acc
    return (p - 2.0 ** f) / 2.0 ** f


def horner_fp32(a32, f):
    f = f.astype(np.float32)
    acc = np.float32(a32[-1]) * np.ones_like(f)
    for c in a32[-2::-1]:
        acc = (acc * f + np.float32(c)).astype(np.float32)
    return (np.float32(1.0) + f * acc).astype(np.float32)


if __name__ == "__main__":
    a = fit(3)
    a32 = np.array(a, dtype=np.float32)
    f = np.linspace(0.0, 1.0, 1 << 20, endpoint=False)
    e64 = np.abs(rel_err(a, f)).max()
    e32 = np.abs(horner_fp32(a32, f).astype(np.float64) / 2.0 ** f - 1).max()
    for i, c in enumerate(a32, 1):
        print(f"a{i} = {float(c)!r:>24}f  ({np.float32(c).view(np.uint32):#010x})")
    print(f"max relative error: {e64:.3e} (fp64 coefficients), {e32:.3e} (fp32 Horner)")
