"""The FMA-pipe 2^x of the attention kernel: its coefficients are the ones
the committed derivation produces, and their float32 evaluation stays within
1e-7 relative of 2^f on [-1/2, 1/2] (about the accuracy of the MUFU ex2)."""
import os
import re

import numpy as np

from bit_quantization_b200.csrc import fit_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _kernel_coefficients():
    src = open(os.path.join(ROOT, "bit_quantization_b200", "csrc", "attn.cuh")).read()
    body = src[src.index("float exp2_fma(float x)"):]
    body = body[:body.index("}")]
    nums = [float(x) for x in re.findall(r"([0-9.]+e[-+][0-9]+)f", body)]
    # q starts at the top coefficient; each fmaf adds the next lower one; the last is 1.0f
    return np.array(nums[::-1] and [1.0] + nums[::-1], np.float32)


def test_coefficients_match_derivation():
    c = fit_exp2.coefficients()
    k = _kernel_coefficients()
    assert len(k) == len(c)
    assert np.array_equal(k, c)


def test_error_bound():
    assert fit_exp2.max_rel_error(fit_exp2.coefficients()) < 1e-7


def test_range_reduction_reassembles_exactly():
    # 2^n * p(f) with n = round(x): exponent arithmetic is exact, so the
    # relative error over x in [-125, 0] is the polynomial's.
    c = fit_exp2.coefficients()
    x = np.linspace(-125, 0, 400001).astype(np.float32)
    n = np.rint(x.astype(np.float64))
    f = (x.astype(np.float64) - n).astype(np.float32)
    y = np.ldexp(fit_exp2.horner_f32(c, f).astype(np.float64), n.astype(int))
    assert np.max(np.abs(y / np.exp2(x.astype(np.float64)) - 1)) < 1e-7
