"""Fits the polynomial the softmax kernels use for part of their exp2 work.

    python -m io_aware_attention_02_b200.fit_exp2_poly [--degree 3]

2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2].  The factor
2^j goes into the exponent bits with one integer shift-add; 2^f is
approximated by the polynomial p(f) = c0 + c1 f + ... + cn f^n that minimises
the maximum RELATIVE error max |p(f) / 2^f - 1| on [-1/2, 1/2].  The
coefficients come from the Remez exchange algorithm (E. Ya. Remez, 1934):
solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on n + 2 reference points, move the
points to the extrema of the weighted error, repeat until the extrema
equioscillate.  The fit runs in float64 and the result is rounded to fp32,
the precision the kernel evaluates it in.

This script is the source of the coefficients of exp2_poly2 in
csrc/fwd_sm100.cuh (degrees 3 and 2); it prints them together with the
achieved error bound.  tests/test_exp2_poly.py checks that the kernel's
literals are this fit rounded to fp32.
"""

from __future__ import annotations

import argparse

import numpy as np


def remez_exp2(degree: int, iters: int = 40):
    n = degree
    lo, hi = -0.5, 0.5
    # initial reference: Chebyshev extrema mapped to [lo, hi]
    k = np.arange(n + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(lo, hi, 200001)
    coef, E = None, None
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, : n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** xi
        b = 2.0 ** x
        sol = np.linalg.solve(A, b)
        coef, E = sol[: n + 1], sol[n + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the n + 2 alternating extrema of err
        s = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n + 2:
            break
        # keep the n + 2 largest consecutive alternations
        while len(idx) > n + 2:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        x_new = grid[idx]
        if np.allclose(x_new, x, atol=1e-12):
            break
        x = x_new
    return coef, abs(E)


def fp32_error(coef32: np.ndarray) -> float:
    """Max relative error of the fp32 Horner evaluation on a dense grid."""
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        p = (p * f + c).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--degree", type=int, default=3)
    a = ap.parse_args()
    coef, E = remez_exp2(a.degree)
    c32 = coef.astype(np.float32)
    print(f"degree {a.degree}: minimax relative error {E:.3e}; fp32 evaluation {fp32_error(c32):.3e}")
    for i, c in enumerate(c32):
        print(f"  c{i} = {float(c)!r}f  // 0x{c.view(np.uint32):08x}")


if __name__ == "__main__":
    main()
