"""The attention parity bar shared by the GPU tests (prefill and decode).

Bar (max-abs 1e-2 and cosine >= 0.9999 against the oracle's emulation of
the same quantisation and tiling), element by element against
the oracle's fp64 result before its final rounding:

    |got - want| <= 1e-2 + half an ulp of the 16-bit output type at want
                         + tol

where `tol` is the oracle's bound for roundings that are not unique: a
probability whose E2M1 code, UE4M3 block scale or 16-bit value lies within
the GPU arithmetic's error of a rounding midpoint may take either rounding
(the bound and its pins: tests/test_oracle_tol_pins.py).  The bar leans on
`tol` only where an element exceeds 1e-2 + half an ulp; such elements must
have tol > 0 (a real midpoint in their row) and be rare: at most
MAX_TOL_RELIANCE of the compared elements.  Every comparison prints how many
elements have tol > 0, the largest tol and how many needed it.
"""
import numpy as np
import torch

MAX_ABS = 1e-2
MIN_COS = 0.9999
MAX_TOL_RELIANCE = 1e-3


def half_ulp(x, dtype):
    """Half the spacing of the 16-bit type at |x| (subnormal floor included)."""
    mant, emin = (7, -126) if dtype == torch.bfloat16 else (10, -14)
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** emin)))
    return 0.5 * 2.0 ** (e - mant)


def compare(got, want64, dtype, tol=None, what="out"):
    """Applies the bar; returns (max abs error, cosine, stats)."""
    got = np.asarray(got, np.float64).reshape(-1)
    want = np.asarray(want64, np.float64).reshape(-1)
    tol = np.zeros_like(want) if tol is None else np.asarray(tol, np.float64).reshape(-1)
    excess = np.abs(got - want) - half_ulp(want, dtype)
    over = excess > MAX_ABS            # elements that pass only through tol, if at all
    n = want.size
    nrm = np.linalg.norm(got) * np.linalg.norm(want)
    cos = float(got @ want / nrm) if nrm > 0 else 1.0
    stats = {"elements": n, "tol_nonzero": int(np.count_nonzero(tol)),
             "tol_max": float(tol.max()) if n else 0.0, "need_tol": int(over.sum()),
             "max_excess": float(excess.max()) if n else 0.0}
    print(f"\n[parity] {what}: {n} elements, tol > 0 on {100 * stats['tol_nonzero'] / max(n, 1):.1f}%"
          f" (max {stats['tol_max']:.2e}), {stats['need_tol']} over 1e-2 + ulp/2 "
          f"({100 * stats['need_tol'] / max(n, 1):.4f}%), max excess {stats['max_excess']:.2e}, "
          f"cos {cos:.6f}")
    worst = int(np.argmax(excess - tol)) if n else 0
    assert n == 0 or excess[worst] - tol[worst] <= MAX_ABS, (
        f"{what}: |err| - ulp/2 - tol = {excess[worst] - tol[worst]:.3e} at {worst} (got "
        f"{got[worst]}, want {want[worst]}, tol {tol[worst]:.3e})")
    assert cos >= MIN_COS, f"{what}: cosine {cos:.6f}"
    assert np.all(tol[over] > 0), f"{what}: elements over the bar without a non-unique rounding"
    assert over.sum() <= MAX_TOL_RELIANCE * n, (
        f"{what}: {int(over.sum())} of {n} elements pass only through tol")
    return float(np.max(np.abs(got - want))) if n else 0.0, cos, stats
