"""Coefficients of the FMA-pipe exp2 used for part of the softmax
probabilities of the attention kernel (csrc/attn.cuh, `exp2_fma2`).

Method: range reduction x = n + f with n = round(x) (Cody-Waite style, by
adding and subtracting 1.5 * 2^23 in fp32), so f is in [-1/2, 1/2] and
2^x = 2^n * 2^f, the power 2^n added to the exponent field as an integer;
2^f by a degree-4 polynomial that interpolates 2^f exactly at five nodes.
Four nodes are fixed by what the probabilities feed: the E2M1 code of
t = 2^x changes where t crosses a rounding midpoint of the E2M1 grid
(0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5), i.e. where f crosses
0, log2(1.5) - 1, log2(1.25), log2(1.75) - 1; interpolating there makes the
polynomial's codes those of the exact exponential up to fp32 evaluation
rounding (the polynomial is increasing, so it cannot cross a midpoint
elsewhere).  The fifth node is placed to minimise the largest relative
error on [-1/2, 1/2], which only the row sum of the probabilities sees.

    python -m bit_quantization_b200.fit_exp2     # prints the coefficients
"""
import numpy as np

# fractional positions (after rounding x to the nearest integer) where
# 2^x crosses an E2M1 rounding midpoint
THRESHOLD_NODES = (0.0, np.log2(1.5) - 1.0, np.log2(1.25), np.log2(1.75) - 1.0)


def interpolant(nodes):
    """Monomial coefficients c0..c4 of the quartic through 2^f at the nodes."""
    A = np.vander(np.asarray(nodes, np.float64), 5, increasing=True)
    return np.linalg.solve(A, np.exp2(np.asarray(nodes, np.float64)))


def max_rel_error(c, grid=np.linspace(-0.5, 0.5, 20001)):
    p = np.polynomial.polynomial.polyval(grid, c)
    return float(np.max(np.abs(p / np.exp2(grid) - 1.0)))


def fit():
    """(coefficients, fifth node, max relative error in exact arithmetic)."""
    best = None
    for t5 in np.linspace(-0.5, 0.5, 2001):
        if min(abs(t5 - n) for n in THRESHOLD_NODES) < 0.02:
            continue
        c = interpolant(THRESHOLD_NODES + (t5,))
        e = max_rel_error(c)
        if best is None or e < best[2]:
            best = (c, float(t5), e)
    return best


def coefficients_f32():
    c, _, _ = fit()
    return [float(np.float32(x)) for x in c]


if __name__ == "__main__":
    c, t5, e = fit()
    print(f"fifth node {t5:.4f}, max relative error {e:.3e}")
    for i, x in enumerate(c):
        print(f"c{i} = {np.float32(x)!r}  ({x:.17g})")
