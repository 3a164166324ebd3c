"""Coefficients of the polynomial 2^f that the kernels evaluate on the FMA pipe.

The softmax needs 2^x for every score.  The special-function unit (MUFU
``ex2``) does 16 of them per clock per SM, half the rate the tensor cores need
at head dim 64, so the kernels compute a share of them on the FP32 pipe instead:
x = n + f with n = round(x) and f in [-1/2, 1/2], 2^f from a polynomial, and n
added to the exponent field.

This script fits that polynomial: degree 3, least maximum RELATIVE error on
[-1/2, 1/2], by the Remez exchange algorithm (Remez 1934; e.g. Cheney,
"Introduction to Approximation Theory", ch. 3) on the weighted error
(p(f) - 2^f) / 2^f.  It then rounds the coefficients to fp32 and measures the
error of the fp32 Horner evaluation on a dense grid.

Run ``python -m causal_attention_fwd_b200.exp2_fit`` to print the constants; a
CPU test checks that the values in ``csrc/sm100_ptx.cuh`` are the ones it
produces and that the error bound holds.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _err(c, f):
    """Relative error of the polynomial with coefficients c (c[0] + c[1] f + ...)."""
    return np.polyval(c[::-1], f) / np.exp2(f) - 1.0


def remez(degree: int = DEGREE, iters: int = 60) -> np.ndarray:
    n = degree
    # start from the Chebyshev extrema mapped to [LO, HI]
    k = np.arange(n + 2)
    x = (LO + HI) / 2 + (HI - LO) / 2 * -np.cos(np.pi * k / (n + 1))
    grid = np.linspace(LO, HI, 200001)
    c = np.zeros(n + 1)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i for the coefficients and E
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, : n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * np.exp2(xi)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[: n + 1]
        e = _err(c, grid)
        # new reference: one extremum of the error per sign-alternating segment
        sign = np.sign(e)
        sign[sign == 0] = 1
        cuts = np.flatnonzero(np.diff(sign)) + 1
        segs = np.split(np.arange(grid.size), cuts)
        ext = [s[np.argmax(np.abs(e[s]))] for s in segs]
        if len(ext) < n + 2:
            break
        # keep the n + 2 largest consecutive alternating extrema
        ext = np.array(ext)
        while ext.size > n + 2:
            if abs(e[ext[0]]) < abs(e[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x_new = grid[ext]
        if np.allclose(x_new, x, atol=1e-12, rtol=0):
            break
        x = x_new
    return c


def fp32_coefficients() -> np.ndarray:
    return remez().astype(np.float32)


def _fma32(a, b, c):
    """fp32 fused multiply-add: a*b is exact in float64 for fp32 a, b."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def eval_fp32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """The kernels' Horner evaluation in fp32: ((c3 f + c2) f + c1) f + c0."""
    f = f.astype(np.float32)
    p = np.full_like(f, c32[3])
    for k in (2, 1, 0):
        p = _fma32(p, f, np.full_like(f, c32[k]))
    return p


def exp2_emulated(x: np.ndarray, c32: np.ndarray, clamp: float = -126.0) -> np.ndarray:
    """The whole fp32 emulation of 2^x as the kernels run it (x <= 64): clamp,
    round by the 1.5*2^23 addition, Horner, exponent add."""
    x = np.maximum(x.astype(np.float32), np.float32(clamp))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = eval_fp32(c32, f)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def max_rel_error(c32: np.ndarray, n: int = 2000001) -> float:
    f = np.linspace(LO, HI, n).astype(np.float32)
    return float(np.max(np.abs(eval_fp32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fp32_coefficients()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v):.9g}f  (bits {np.float32(v).view(np.uint32):#010x})")
    print(f"max relative error of the fp32 evaluation on [-1/2, 1/2]: {max_rel_error(c):.3e}")
