"""Fits the polynomial of the FMA-pipe exponential in tc_primitives.cuh.

The tensor-core softmax kernels compute part of their exponentials 2^x without
the SFU: x = j + f with j = rint(x) and f in [-1/2, 1/2] (the Cody-Waite
split, exact in fp32 for |x| < 2^22), 2^f from a degree-3 polynomial p(f), and
2^j by adding j to the exponent field of p(f).  This script finds p by the
Remez exchange for the smallest maximum RELATIVE error of p(f) against 2^f on
[-1/2, 1/2], rounds the coefficients to fp32 and reports the error of the
fp32 Horner evaluation (the form the kernels use) on a dense grid.

    python efficient_vision_attention_b200/csrc/fit_exp2_poly.py [degree]

Output: the coefficients c0..cn (p(f) = c0 + c1 f + ... + cn f^n) as fp32
hexadecimal literals and the measured maximum relative error.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_relative(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40) -> np.ndarray:
    """Minimax polynomial of degree deg for 2^f on [lo, hi] in relative error."""
    n = deg + 2                                   # equioscillation points
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for the coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:deg + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference points: the extrema of the error between sign changes
        sgn = np.sign(err)
        cuts = np.flatnonzero(np.diff(sgn) != 0) + 1
        segs = np.split(np.arange(grid.size), cuts)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) < n:
            break
        # keep n alternating extrema with the largest magnitudes
        while len(ext) > n:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[ext]
    return coef


def fp32_horner_error(coef32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    p = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        p = (p * f + c).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main() -> None:
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef = remez_relative(deg)
    c32 = coef.astype(np.float32)
    for i, c in enumerate(c32):
        bits = int(np.frombuffer(c.tobytes(), dtype=np.uint32)[0])
        print(f"c{i} = {float(c):.9g}f   // 0x{bits:08x}")
    print(f"max relative error of the fp32 Horner form on [-1/2, 1/2]: "
          f"{fp32_horner_error(c32):.3e}")


if __name__ == "__main__":
    main()
