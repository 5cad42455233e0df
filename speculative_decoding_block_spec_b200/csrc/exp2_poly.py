"""Coefficients of the polynomial 2^f on [-1/2, 1/2] used by exp2_fma() in
exp2_fma.cuh, and their error.

    python speculative_decoding_block_spec_b200/csrc/exp2_poly.py [degree]

Method: the Remez exchange algorithm (E. Ya. Remez, 1934) for the polynomial
p of the given degree that minimises the maximum RELATIVE error
|p(f) / 2^f - 1| over [-1/2, 1/2]. Each iteration solves the linear system
p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i} on degree + 2 reference points, then
moves the reference to the extrema of the weighted error. The computation is
in float64 on a dense grid; the printed coefficients are then rounded to
float32, which is what the kernel evaluates (in Horner form with fused
multiply-adds), and the script reports the relative error of the rounded
polynomial in exact (float64) evaluation.
"""
import sys

import numpy as np


def remez_exp2(degree, iters=30, grid=200001):
    a, b = -0.5, 0.5
    xs = np.linspace(a, b, grid)
    n = degree + 2
    # initial reference: Chebyshev extrema
    ref = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    coef = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], xs) / 2.0 ** xs - 1.0
        # new reference: one extremum of the error per sign-alternating segment
        sign = np.sign(err)
        cuts = np.flatnonzero(np.diff(sign) != 0) + 1
        segs = np.split(np.arange(grid), cuts)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs if len(s)]
        if len(ext) < n:
            break
        # keep the n largest alternating extrema
        while len(ext) > n:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext.pop(drop)
        ref = xs[ext]
    return coef


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c = remez_exp2(degree)
    c32 = c.astype(np.float32)
    xs = np.linspace(-0.5, 0.5, 1000001)
    err64 = np.max(np.abs(np.polyval(c[::-1], xs) / 2.0 ** xs - 1.0))
    err32 = np.max(np.abs(np.polyval(c32.astype(np.float64)[::-1], xs) / 2.0 ** xs - 1.0))
    print("degree %d: max relative error %.3e (float64 coefficients), %.3e (float32 coefficients)"
          % (degree, err64, err32))
    for k, v in enumerate(c32):
        print("  c%d = %.9ef  (0x%08x)" % (k, float(v), np.float32(v).view(np.uint32)))


if __name__ == "__main__":
    main()
