"""Minimax polynomial for 2^f on [-1/2, 1/2] (relative error), by the Remez
exchange algorithm (E. Ya. Remez, 1934).

The forward kernel evaluates part of its exp2 on the FMA pipe instead of the
MUFU unit: x = j + f with j = rint(x) (by the 1.5 * 2^23 rounding trick),
2^f ~ p(f) with p of degree 3, and 2^j applied by adding j to the exponent
bits. This script computes p's coefficients (float64 Remez iteration,
then rounded to float32) and the worst relative error of the float32
evaluation; the kernel's constants are the printed values.

    python -m sparse_long_sequence_dilated_b200.csrc.fit_exp2_poly
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    n = degree
    # start from Chebyshev extrema
    k = np.arange(n + 2)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^{x_i} (1 + (-1)^i E) = 0  ->  sum_k c_k x_i^k - (-1)^i E 2^{x_i} = 2^{x_i}
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        idx = []
        sign = np.sign(err)
        start = 0
        for j in range(1, len(grid) + 1):
            if j == len(grid) or sign[j] != sign[start]:
                seg = slice(start, j)
                idx.append(start + int(np.argmax(np.abs(err[seg]))))
                start = j
        if len(idx) < n + 2:
            break
        # keep the n + 2 largest alternating extrema
        while len(idx) > n + 2:
            vals = np.abs(err[idx])
            if vals[0] < vals[-1]:
                idx.pop(0)
            else:
                idx.pop()
        x = grid[idx]
    return c


def eval_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """Horner in float32 with fused multiply-add rounding emulated per step."""
    f = f.astype(np.float32)
    acc = np.float32(c32[-1]) * np.ones_like(f)
    for ck in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return acc


def main():
    c = remez()
    c32 = c.astype(np.float32)
    f = np.linspace(LO, HI, 1000001)
    rel = np.abs(eval_f32(c32, f).astype(np.float64) / 2.0 ** f - 1.0)
    for i, ck in enumerate(c32):
        print(f"c{i} = {float(ck):.9e}f")
    print(f"max relative error (float32 evaluation) = {rel.max():.3e}")


if __name__ == "__main__":
    main()
