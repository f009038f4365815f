"""Fits the polynomial that attention.cu uses for 2^f, f in [-1/2, 1/2], on the FMA pipe.

    python resolution_vit_vision_b200/csrc/fit_exp2_poly.py [degree]

Method: the Remez exchange algorithm for the best uniform (minimax) approximation, applied to the
relative error p(f) / 2^f - 1 (weight 2^-f). Start from the Chebyshev extrema; each round solves
p(x_i) - 2^x_i = (-1)^i E 2^x_i on the n + 2 reference points, then moves every reference point to
the extremum of the error in its interval, until the levelled error E stops changing. The fitted
coefficients are then rounded to float32 and the relative error of the float32 Horner evaluation
(one fused multiply-add per step, as on the GPU) is measured on a dense grid. attention.cu holds
the float32 coefficients this prints for degree 3, and the kernel's range reduction
x = j + f, j = rint(x), makes the relative error of 2^x that of 2^f.
"""
from __future__ import annotations

import sys

import numpy as np


def remez(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = deg + 2
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * -np.cos(np.pi * k / (n - 1))      # Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    E = 0.0
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extremum of the error inside each sign-constant stretch
        s = np.sign(err)
        cuts = np.nonzero(np.diff(s))[0] + 1
        parts = np.split(np.arange(grid.size), cuts)
        ext = [p[np.argmax(np.abs(err[p]))] for p in parts if p.size]
        if len(ext) < n:
            break
        while len(ext) > n:                                   # keep the n largest, alternating
            drop = min(range(len(ext)), key=lambda i: abs(err[ext[i]]))
            ext.pop(drop)
        x = grid[np.array(ext)]
    return c, abs(E)


def f32_horner_error(c32: np.ndarray, n: int = 2_000_001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        # fused multiply-add: one rounding of the exact p * f + ck
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, E = remez(deg)
    c32 = c.astype(np.float32)
    print(f"degree {deg}: levelled relative error {E:.4e}; float32 Horner max relative error "
          f"{f32_horner_error(c32):.4e}")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci)!r}f  ({ci.view(np.uint32):#010x})")
