"""Fit the polynomial the attention kernel uses to evaluate 2^f on the FMA pipe.

Method: Remez exchange (E. Remez, 1934) for the minimax *relative* error of a
degree-n polynomial p(f) ~ 2^f on [-1/2, 1/2]:

  1. start from the Chebyshev extrema as n+2 reference points x_i;
  2. solve the linear system  p(x_i) - 2^{x_i} = (-1)^i * E * 2^{x_i}
     for the n+1 coefficients and the levelled error E;
  3. move the reference points to the local extrema of the weighted error
     e(f) = p(f) / 2^f - 1 and repeat until the extrema are level.

Range reduction (Cody and Waite's argument split, which is exact for base 2):
x = j + f with j = round(x) taken by adding 1.5 * 2^23 in float32 (round to
nearest), so |f| <= 1/2 and f = x - j has no rounding error; then
2^x = 2^j * p(f), with 2^j applied by adding j to the float32 exponent field.

Running this script prints the float32 coefficients and the worst relative
error of the float32 Horner evaluation over a dense grid. The degree-2 and
degree-3 values it printed (`--degree 2`, `--degree 3`) are written into
attn_fwd.cu (exp2_coef; degree 2 is used, since P is rounded to bf16
there). The fp32-mode kernel takes every exponential from MUFU; a degree-5
fit (`--degree 5`) would match MUFU's ~2^-22 if it needed one.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int = 3, iters: int = 30):
    n = degree
    lo, hi = -0.5, 0.5
    k = np.arange(n + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * -np.cos(np.pi * k / (n + 1))
    grid = np.linspace(lo, hi, 200001)
    coef = None
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        for i, xi in enumerate(x):
            A[i, : n + 1] = xi ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[: n + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # local extrema of the error, including the interval ends
        idx = [0]
        for i in range(1, grid.size - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0 and abs(err[i]) > 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        # keep n+2 alternating extrema of largest magnitude
        cand = [(grid[i], err[i]) for i in idx]
        merged = []
        for xv, ev in cand:
            if merged and np.sign(merged[-1][1]) == np.sign(ev):
                if abs(ev) > abs(merged[-1][1]):
                    merged[-1] = (xv, ev)
            else:
                merged.append((xv, ev))
        while len(merged) > n + 2:
            if abs(merged[0][1]) < abs(merged[-1][1]):
                merged.pop(0)
            else:
                merged.pop()
        if len(merged) < n + 2:
            break
        x = np.array([m[0] for m in merged])
    return coef


def f32_horner(c32, f):
    p = np.float32(c32[-1])
    for c in c32[-2::-1]:
        p = (p * f + np.float32(c)).astype(np.float32)
    return p


def check(coef, degree):
    c32 = np.asarray(coef, dtype=np.float32)
    x = np.linspace(-24.0, 8.0, 2_000_001).astype(np.float32)
    magic = np.float32(1.5 * 2 ** 23)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = f32_horner(c32, f)
    bits = p.view(np.uint32).astype(np.int64) + (t.view(np.uint32).astype(np.int64) << 23)
    y = (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    return c32, float(rel.max())


if __name__ == "__main__":
    import sys

    degrees = [int(sys.argv[sys.argv.index("--degree") + 1])] if "--degree" in sys.argv else [3]
    for deg in degrees:
        c = remez_exp2(deg)
        c32, worst = check(c, deg)
        print(f"degree {deg}: " + ", ".join(f"{v:.9e}f" for v in c32) + f"   max rel err {worst:.3e}")
