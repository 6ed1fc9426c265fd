"""Derives the coefficients of the FMA-pipe 2^f used by the attention kernel.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in [-1/2, 1/2];
p is the degree-6 polynomial interpolating 2^f at the seven Chebyshev nodes of
[-1/2, 1/2] (near-minimax).  Run it to print the float32 coefficients (lowest
degree first) and the maximum relative error of their float32 Horner
evaluation with fused multiply-adds.
"""
import numpy as np

DEG = 6


def coefficients():
    k = np.arange(DEG + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (DEG + 1)))
    c = np.linalg.solve(np.vander(nodes, DEG + 1, increasing=True), np.exp2(nodes))
    return c.astype(np.float32)


def horner_f32(c, f):
    """Float32 Horner with each fused multiply-add rounded once."""
    p = np.full(f.shape, c[-1], np.float32)
    for ci in c[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ci)).astype(np.float32)
    return p


def max_rel_error(c, n=2_000_001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    return float(np.max(np.abs(horner_f32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)))


if __name__ == "__main__":
    c = coefficients()
    print("coefficients:", ", ".join(f"{float(x):.17g}" for x in c))
    print("max relative error:", max_rel_error(c))
