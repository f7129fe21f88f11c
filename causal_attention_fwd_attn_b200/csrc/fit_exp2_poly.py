"""Fits the polynomial behind exp2_poly2 (sm100_ptx.cuh): p(f) ~ 2^f on [-1/2, 1/2],
minimising the maximum relative error by the Remez exchange algorithm, and prints
the coefficients rounded to fp32 with the error of fp32 Horner evaluation.

    python causal_attention_fwd_attn_b200/csrc/fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_exp2(deg, a=-0.5, b=0.5, iters=30, grid=200001):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    g = np.linspace(a, b, grid)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the reference points
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * 2.0 ** x[i]
        c = np.linalg.solve(A, 2.0 ** x)[:deg + 1]
        err = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        ext = [0] + [i for i in range(1, grid - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [grid - 1]
        alt = []
        for i in ext:  # alternating extrema, keeping the larger of same-sign neighbours
            if alt and np.sign(err[i]) == np.sign(err[alt[-1]]):
                if abs(err[i]) > abs(err[alt[-1]]):
                    alt[-1] = i
            else:
                alt.append(i)
        while len(alt) > n:
            alt.pop(0 if abs(err[alt[0]]) < abs(err[alt[-1]]) else -1)
        x = g[alt]
    return c


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c32 = remez_exp2(deg).astype(np.float32)
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) - 2.0 ** f.astype(np.float64)) / 2.0 ** f.astype(np.float64)
    print(f"degree {deg}: max relative error (fp32 Horner) {rel.max():.3g}")
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v).hex()}")


if __name__ == "__main__":
    main()
