"""Fit the polynomial the kernel uses for 2^f on f in [-1/2, 1/2].

The kernel evaluates part of the softmax exponentials on the FMA pipe:
2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2] (range
reduction for base 2 is exact); 2^j goes into the exponent field with one
integer add, and 2^f is a polynomial.  This script fits that polynomial by
the Remez exchange algorithm on the *relative* error (weight 1 / 2^f),
rounds the coefficients to fp32, and reports the worst relative error of the
fp32 Horner evaluation on a dense grid.

    python gen_exp2_poly.py [degree]
"""

import sys

import numpy as np


def remez_relative(degree: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    n = degree + 2
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # solve  sum_i c_i x^i - 2^x = (-1)^k E 2^x   at the reference points
        A = np.zeros((n, n))
        for r in range(n):
            A[r, :degree + 1] = x[r] ** np.arange(degree + 1)
            A[r, degree + 1] = -((-1.0) ** r) * 2.0 ** x[r]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.where(np.diff(sign) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            seg = np.abs(err[a:b])
            ext.append(a + int(np.argmax(seg)))
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest magnitude
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext.pop(0)
            else:
                ext.pop()
        x = grid[np.array(ext)]
    return coef


def fp32_horner(coef32, f):
    f = f.astype(np.float32)
    acc = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        # fma in fp64 then round to fp32 models a fused multiply-add
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(c)).astype(np.float32)
    return acc


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = remez_relative(degree)
    coef32 = coef.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001)
    p = fp32_horner(coef32, f).astype(np.float64)
    rel = np.max(np.abs(p - 2.0 ** f) / 2.0 ** f)
    print(f"degree {degree}: max relative error {rel:.3e} ({np.log2(rel):.2f} bits)")
    for i, c in enumerate(coef32):
        print(f"  c{i} = {float(c)!r}f  (0x{np.float32(c).view(np.uint32):08x})")


if __name__ == "__main__":
    main()
