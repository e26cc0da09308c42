"""Fits the polynomial of msa_exp2.cuh: p(f) ~ 2^f on [-1/2, 1/2] with the
smallest largest RELATIVE error (Remez exchange on the equioscillation
system p(x_i) - 2^x_i = (-1)^i E 2^x_i), then rounds the coefficients to fp32
and reports the error of the fp32 Horner evaluation with fused multiply-adds.

    python block_sparse_long_exp_b200/csrc/exp2_poly_fit.py [degree]

prints the coefficients as C hexadecimal float literals, lowest order first.
"""
import sys

import numpy as np


def remez(deg, lo=-0.5, hi=0.5, iters=40, grid=400001):
    m = deg + 2
    x = 0.5 * (lo + hi) - 0.5 * (hi - lo) * np.cos(np.pi * np.arange(m) / (m - 1))
    g = np.linspace(lo, hi, grid)
    for _ in range(iters):
        y = 2.0 ** x
        A = np.empty((m, m))
        for i in range(deg + 1):
            A[:, i] = x ** i
        A[:, deg + 1] = (-1.0) ** np.arange(m) * y
        c = np.linalg.solve(A, y)[:deg + 1]
        err = np.polyval(c[::-1], g) / 2.0 ** g - 1.0
        # one extremum per run of constant sign: the new reference points
        cuts = np.concatenate([[0], np.nonzero(np.diff(np.sign(err)))[0] + 1, [grid]])
        ext = [a + int(np.argmax(np.abs(err[a:b]))) for a, b in zip(cuts[:-1], cuts[1:])]
        if len(ext) > m:
            ext = sorted(sorted(ext, key=lambda j: -abs(err[j]))[:m])
        if len(ext) < m:
            break
        x = g[ext]
    return c


def fp32_horner_error(c32, lo=-0.5, hi=0.5, n=1 << 20):
    """Largest relative error of the fp32 evaluation (each fma rounded once)."""
    f = np.linspace(lo, hi, n).astype(np.float32).astype(np.float64)
    p = np.full_like(f, np.float64(c32[-1]))
    for ci in c32[-2::-1]:
        p = (p * f + np.float64(ci)).astype(np.float32).astype(np.float64)
    return float(np.max(np.abs(p / 2.0 ** f - 1.0)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c32 = remez(deg).astype(np.float32)
    print(f"degree {deg}: largest relative error of the fp32 evaluation {fp32_horner_error(c32):.3e}")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci).hex()}f  /* {float(ci):.9g} */")


if __name__ == "__main__":
    main()
