"""The FMA-pipe exp2 of the attention kernel (exp2_fma2 in csrc/attn.cuh),
emulated step for step in fp32 on the CPU: its constants are those the fit
script derives, it stays within 2e-5 relative of 2^x, it is increasing, it
gives the E2M1 codes of the exact exponential except within a few fp32 ulps
of a rounding midpoint (where it interpolates), and it returns a tiny
non-negative value for arguments at or below -126 (masked scores are -inf).
The E2M1 codes come from the oracle's encoder."""
import os
import re

import numpy as np

from bit_quantization_b200 import fit_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
M = np.float32(12582912.0)


def _f32(x):
    return np.asarray(x, np.float32)


def _fma(a, b, c):
    # fp32 fused multiply-add: the product is exact in fp64, one rounding
    # to fp32 after the add (a double rounding only on exact fp64 ties)
    return _f32(np.float64(a) * np.float64(b) + np.float64(c))


def emulate(x):
    c = [np.float32(v) for v in fit_exp2.coefficients_f32()]
    x = np.maximum(_f32(x), np.float32(-126.0))
    j = _f32(x + M)
    n = _f32(j - M)
    f = _fma(n, np.float32(-1.0), x)
    p = _fma(c[4], f, c[3])
    p = _fma(p, f, c[2])
    p = _fma(p, f, c[1])
    p = _fma(p, f, c[0])
    bits = p.view(np.uint32).astype(np.uint64) + (j.view(np.uint32).astype(np.uint64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_constants_match_the_fit():
    src = open(os.path.join(ROOT, "bit_quantization_b200", "csrc", "attn.cuh")).read()
    got = [float(np.float32(v)) for v in re.findall(r"kExp2C\d = ([0-9.e-]+)f", src)]
    assert got == fit_exp2.coefficients_f32()[1:]
    assert fit_exp2.coefficients_f32()[0] == 1.0


def test_relative_error_and_monotone():
    x = np.linspace(-125.0, 3.0, 2_000_001).astype(np.float32)
    t = emulate(x).astype(np.float64)
    rel = np.abs(t / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 2e-5, rel.max()
    assert np.all(np.diff(t) >= 0.0)


def test_codes_of_the_exact_exponential(orc):
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rng = np.random.default_rng(3)
    xs = [rng.uniform(-6.0, 3.0, 400_000)]
    for m in mids:  # dense around every midpoint
        xs.append(np.log2(m) + rng.uniform(-1e-3, 1e-3, 50_000))
    x = np.concatenate(xs).astype(np.float32)
    t = emulate(x)
    exact = np.exp2(x.astype(np.float64))
    near = np.min(np.abs(exact[:, None] / mids[None, :] - 1.0), axis=1) < 4e-7
    got = orc.e2m1_encode(t)
    want = orc.e2m1_encode(exact.astype(np.float32))
    assert np.array_equal(got[~near], want[~near])
    assert (~near).sum() > 700_000


def test_clamped_arguments():
    t = emulate(np.array([-np.inf, -1e30, -1000.0, -126.0, -125.6], np.float32))
    assert np.all(np.isfinite(t)) and np.all(t >= 0.0) and np.all(t <= 2.0 ** -125)
