"""Coefficients of the FMA-pipe exp2 used by the attention softmax.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]: for base 2
the reduction is exact in fp32 (n and f are both representable), so no
multi-word constant is needed as in a Cody-Waite reduction for e^x.  2^f is a
degree-4 polynomial p(f) chosen by the Remez exchange algorithm to minimise
the maximum RELATIVE error |p(f) / 2^f - 1| on [-1/2, 1/2] (equioscillation
at 6 points).  The kernel evaluates p in fp32 by Horner's rule with fused
multiply-adds and adds n to the exponent field.

  python -m score_keys_pooled_b200.csrc.exp2_poly   # prints the coefficients

The printed values are the ones in sparse_attn2.cuh (kExp2C0..kExp2C4);
tests/test_exp2_poly.py checks both that and the fp32 evaluation's error.
"""
from __future__ import annotations

import math

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    """Minimax relative-error polynomial for 2^f on [LO, HI]; returns
    (coefficients c0..c_degree in fp64, levelled error E)."""
    m = degree + 2
    # start from Chebyshev extrema
    k = np.arange(m)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (m - 1))
    E = 0.0
    c = np.zeros(degree + 1)
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_j c_j x_i^j - 2^{x_i} (1 + (-1)^i E) = 0, i.e.
        # sum_j c_j x_i^j - (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum of the error per sign run
        sign = np.sign(err)
        idx = []
        start = 0
        for j in range(1, len(grid) + 1):
            if j == len(grid) or sign[j] != sign[start]:
                seg = np.arange(start, j)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = j
        if len(idx) < m:
            break
        # keep the m largest alternating extrema
        while len(idx) > m:
            a = np.abs(err[idx])
            drop = 0 if a[0] < a[-1] else len(idx) - 1
            idx.pop(drop)
        x = grid[idx]
    return c, abs(E)


def emulate(x: np.ndarray, c32: np.ndarray) -> np.ndarray:
    """The kernel's evaluation in fp32: n by the 1.5 * 2^23 rounding trick, f
    = x - n, Horner with fused multiply-adds (computed exactly in fp64 and
    rounded once to fp32), then n added to the exponent field.  x is clamped
    to [-125, 64] as in the kernel (arguments are <= 8 there)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full(f.shape, c32[-1], dtype=np.float32)
    for cj in c32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(cj)).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, E = remez()
    for j, v in enumerate(c):
        print(f"kExp2C{j} = {float(np.float32(v))!r:>16}f  (fp64 {v!r})")
    print(f"levelled relative error {E:.3e}")
    print(f"check: ln2 = {math.log(2):.10f}, c1 = {c[1]:.10f}")
