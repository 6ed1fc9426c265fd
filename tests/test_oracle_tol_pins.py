"""Pins of the oracle's bound `tol` for roundings that are not unique.

The GPU evaluates the emulation's quantities in another order (fp32
tensor-core accumulation of the scores, fp32 exponent arguments, hardware
exp2 / log2), so a probability whose E2M1 code, UE4M3 block scale or 16-bit
value lies within that arithmetic's error of a rounding midpoint has two
correct roundings ("ThriftAttention", Metodologia step 2: the two-level
quantisation of P; reading R7).  The oracle bounds, per output element, how
far such roundings can move it.  These tests pin that bound against what the
definition fixes, not against its own formula:

* exact zeros: when no probability can sit near a midpoint (all scores equal:
  every P is 1, every code the E2M1 maximum, every block scale exact), the
  bound is exactly 0 on both paths;
* tightness: a probability planted exactly on an E2M1 midpoint in an
  otherwise unambiguous row makes the bound equal, element by element, the
  output change of re-running the emulation with that one code taking the
  other rounding; in the first key tile of a row whose running maximum later
  grows, so the bound must follow the online-softmax rescaling and the final
  division by the row sum;
* soundness: moving every rounding input of the probabilities by a seeded
  random amount within the radius changes an output element by at most its
  bound, and leaves every element whose bound is 0 bit for bit unchanged
  (prefill on both paths, causal, GQA, Hadamard + ScaleSearch, fp16; decode).
"""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import synth


def _case(orc, B, N, H, Hkv, d, blk, causal, frac, ss, had, dtype, seed=0, k_off=3.0, q=None):
    w = synth.AttnWorkload("pin", B, H, Hkv, N, d, dtype, causal, blk, frac, ss, had,
                           k_offset_std=k_off, seed=seed)
    inp = synth.make_attn_inputs(w)
    qq = inp["q"] if q is None else q
    qp, kp, vp = (synth.as_u16(t.reshape(B * N, -1, d)) for t in (qq, inp["k"], inp["v"]))
    cu = np.arange(B + 1, dtype=np.int32) * N
    dt = synth.dtype_code(dtype)

    def run(**hooks):
        with orc.test_hooks(**hooks):
            return orc.thrift_attn(qp, kp, vp, dt, cu, blk, causal, frac, use_ss=ss, use_had=had)
    return run


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_tol_is_zero_when_every_score_is_equal(orc, causal, frac):
    # q = 0: every score is 0, every probability 1 against the running max,
    # the tile maximum 1, the block scales 448 (exact), every code 6 (exact),
    # every 16-bit P exactly 1: nothing is near a rounding midpoint.
    q = torch.zeros((1, 256, 2, 64), dtype=torch.bfloat16)
    run = _case(orc, 1, 256, 2, 1, 64, 64, causal, frac, False, False, torch.bfloat16, q=q)
    r = run()
    assert np.all(r["tol"] == 0.0)
    assert np.all(np.isfinite(r["out64"]))


def _unambiguous_row(r, H, N, d):
    t = r["tol"].reshape(N, H, d)
    for row in range(N):
        if np.all(t[row, 0] == 0.0):
            return row
    return None


@pytest.mark.parametrize("plant_t,force", [(2.5, +1), (np.nextafter(np.float32(2.5), 3), -1),
                                           (0.75, +1), (5.0, +1), (0.25, +1)])
def test_planted_midpoint_bound_equals_the_other_rounding(orc, plant_t, force):
    # Non-causal, 4 key tiles of 64: a code planted in the first tile of a
    # row is rescaled by later growth of the running max and divided by l.
    N, H, d, blk = 256, 1, 64, 64
    run = _case(orc, 1, N, H, 1, d, blk, False, 0.0, False, False, torch.bfloat16, seed=5,
                k_off=0.0)
    base = run()
    row = _unambiguous_row(base, H, N, d)
    assert row is not None
    key = 7  # first key tile
    plant = (0, 0, row, key)
    a = run(plant=plant, plant_t=float(plant_t))
    b = run(plant=plant, plant_t=float(plant_t), force=force)
    ta = a["tol"].reshape(N, H, d)[row, 0]
    oa = a["out64"].reshape(N, H, d)[row, 0]
    ob = b["out64"].reshape(N, H, d)[row, 0]
    moved = np.abs(ob - oa)
    # (a channel whose dequantised value at the planted key is 0 moves by 0)
    assert np.count_nonzero(ta) > d // 2
    # the only ambiguity of the row: the bound is the other rounding's effect
    np.testing.assert_allclose(moved, ta, rtol=1e-9, atol=1e-15)
    # every other row is untouched
    other = np.ones(N, bool)
    other[row] = False
    np.testing.assert_array_equal(a["out64"].reshape(N, H, d)[other],
                                  b["out64"].reshape(N, H, d)[other])


def test_planted_value_away_from_midpoints_adds_nothing(orc):
    # t = 2.0 is an E2M1 value, far from both neighbouring midpoints
    N, H, d, blk = 256, 1, 64, 64
    run = _case(orc, 1, N, H, 1, d, blk, False, 0.0, False, False, torch.bfloat16, seed=5,
                k_off=0.0)
    base = run()
    row = _unambiguous_row(base, H, N, d)
    a = run(plant=(0, 0, row, 7), plant_t=2.0)
    assert np.all(a["tol"].reshape(N, H, d)[row, 0] == 0.0)


PERT_CASES = [
    # B, N, H, Hkv, d, blk, causal, frac, ss, had, dtype
    (1, 384, 2, 1, 128, 128, False, 0.0, False, False, torch.bfloat16),
    (2, 300, 4, 2, 128, 128, True, 0.25, True, True, torch.bfloat16),
    (1, 200, 2, 2, 64, 64, True, 0.5, False, True, torch.float16),
    (1, 256, 2, 2, 64, 128, False, 1.0, False, False, torch.float16),
    (1, 520, 2, 1, 128, 64, True, 0.1, True, False, torch.bfloat16),
]


@pytest.mark.parametrize("case", PERT_CASES, ids=lambda c: "-".join(str(x) for x in c[:10]))
def test_roundings_within_the_radius_stay_within_tol(orc, case):
    run = _case(orc, *case)
    base = run()
    tol, o0 = base["tol"].ravel(), base["out64"].ravel()
    moved_any = 0
    best_ratio = 0.0
    for seed in (1, 2, 3):
        for pert in (1.0, -1.0):
            p = run(pert=pert, seed=seed)
            dlt = np.abs(p["out64"].ravel() - o0)
            assert np.all(dlt <= tol * (1 + 1e-9) + 1e-15), float(np.max(dlt - tol))
            zero = tol == 0.0
            assert np.array_equal(p["out64"].ravel()[zero], o0[zero])
            moved_any += int(np.count_nonzero(dlt))
            nz = tol > 0
            if nz.any():
                best_ratio = max(best_ratio, float(np.max(dlt[nz] / tol[nz])))
    # the perturbations do flip roundings, and the bound is not vacuous
    assert moved_any > 0
    assert best_ratio > 0.3, best_ratio


def test_decode_roundings_within_the_radius_stay_within_tol(orc):
    w = synth.DecodeWorkload("pin", 2, 8, 2, 1024, 300, 1000, 128, torch.bfloat16, 0.25, False)
    inp = synth.make_decode_inputs(w, lengths=[1000, 301])
    q, k, v = (synth.as_u16(inp[n]) for n in ("q", "k", "v"))
    lens = np.array(inp["lengths"], np.int32)
    g_kv = tuple(orc.tensor_scale(np.concatenate(
        [t[b, :L].reshape(-1, 128) for b, L in enumerate(lens)]), 1) for t in (k, v))
    base = orc.thrift_decode(q, k, v, 1, lens, 128, g_kv, w.topk_frac)
    tol, o0 = base["tol"].ravel(), base["out64"].ravel()
    moved = 0
    for seed in (1, 2, 3, 4):
        with orc.test_hooks(pert=1.0 if seed % 2 else -1.0, seed=seed):
            p = orc.thrift_decode(q, k, v, 1, lens, 128, g_kv, w.topk_frac)
        dlt = np.abs(p["out64"].ravel() - o0)
        assert np.all(dlt <= tol * (1 + 1e-9) + 1e-15)
        assert np.array_equal(p["out64"].ravel()[tol == 0.0], o0[tol == 0.0])
        moved += int(np.count_nonzero(dlt))
    assert moved > 0
