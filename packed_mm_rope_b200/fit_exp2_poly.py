"""Fit the degree-3 polynomial used for 2^f, f in [-1/2, 1/2], on the FMA pipe.

Remez exchange (E. Remez, 1934) on the RELATIVE error p(f)/2^f - 1, in
40-digit arithmetic (mpmath), then rounded to fp32; prints the coefficients
c0..c3 used by exp2_fma() in csrc/attention.cuh and the max relative error of
their fp32 Horner evaluation.  Run:  python -m packed_mm_rope_b200.fit_exp2_poly
"""
from __future__ import annotations

import mpmath as mp
import numpy as np


def remez(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 30, grid: int = 4000):
    n = deg + 2
    x = [mp.mpf((a + b) / 2 + (b - a) / 2 * np.cos(np.pi * (n - 1 - i) / (n - 1))) for i in range(n)]
    c, worst = None, None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  -> linear in (c_0..c_deg, E)
        A = mp.matrix(n, n)
        rhs = mp.matrix(n, 1)
        for i, xi in enumerate(x):
            w = mp.power(2, xi)
            for k in range(deg + 1):
                A[i, k] = xi ** k
            A[i, deg + 1] = (-1) ** i * w
            rhs[i] = w
        sol = mp.lu_solve(A, rhs)
        c = [sol[k] for k in range(deg + 1)]

        def err(t):
            return (sum(c[k] * t ** k for k in range(deg + 1)) - mp.power(2, t)) / mp.power(2, t)

        pts = [mp.mpf(a + (b - a) * i / grid) for i in range(grid + 1)]
        vals = [err(t) for t in pts]
        ext = [0] + [i for i in range(1, grid) if (vals[i] - vals[i - 1]) * (vals[i + 1] - vals[i]) <= 0] + [grid]
        merged = []
        for i in ext:
            if merged and mp.sign(vals[merged[-1]]) == mp.sign(vals[i]):
                if abs(vals[i]) > abs(vals[merged[-1]]):
                    merged[-1] = i
            else:
                merged.append(i)
        while len(merged) > n:
            merged.pop(0 if abs(vals[merged[0]]) < abs(vals[merged[-1]]) else -1)
        x = [pts[i] for i in merged]
        worst = max(abs(v) for v in vals)
    return c, float(worst)


def horner_f32_rel_error(c32, samples: int = 200001) -> float:
    t = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    p = np.float32(c32[-1])
    for ck in reversed(c32[:-1]):
        p = (p * t + ck).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / np.exp2(t.astype(np.float64)) - 1).max())


if __name__ == "__main__":
    mp.mp.dps = 40
    coeffs, e = remez(3)
    c32 = [np.float32(float(v)) for v in coeffs]
    for k, v in enumerate(c32):
        print(f"constexpr float EXP2_C{k} = {float(v)!r}f;")
    print(f"# minimax relative error {e:.3e}; fp32 Horner {horner_f32_rel_error(c32):.3e}")
