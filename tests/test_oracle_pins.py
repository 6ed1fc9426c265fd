"""Pins the CPU oracle to facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: values the
pages state (fixtures under tests/golden/), closed forms, invariants, library
routines (numpy / torch / scipy) for the special cases that reduce to them,
and brute force on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

from bit_quantization_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ E2M1

def test_e2m1_grid_matches_golden(orc):
    for code, val in _table("e2m1_grid.txt"):
        got = orc.e2m1_decode([int(code)])[0]
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e2m1_has_15_distinct_values(orc):
    vals = orc.e2m1_decode(np.arange(16))
    assert len(set(float(v) for v in vals)) == 15


def test_e2m1_ties_and_saturation(orc):
    for x, code in _table("e2m1_ties.txt"):
        assert orc.e2m1_encode([float(x)])[0] == int(code), x


def test_e2m1_roundtrip_and_nearest(orc):
    vals = orc.e2m1_decode(np.arange(16))
    assert np.array_equal(orc.e2m1_decode(orc.e2m1_encode(vals)), vals)
    rng = np.random.default_rng(1)
    t = np.concatenate([rng.uniform(-8, 8, 20000), rng.normal(0, 2, 20000)]).astype(np.float32)
    q = orc.e2m1_decode(orc.e2m1_encode(t)).astype(np.float64)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6], np.float64)
    best = np.min(np.abs(t[:, None].astype(np.float64) - grid[None, :]), axis=1)
    assert np.all(np.abs(t - q) == best)
    assert np.all(np.sign(q) * np.sign(t) >= 0)


# ----------------------------------------------------------------- UE4M3

def test_ue4m3_fixed_points(orc):
    for b, val in _table("ue4m3_points.txt"):
        assert orc.ue4m3_decode([int(b)])[0] == float(val)


def test_ue4m3_decode_structure(orc):
    v = orc.ue4m3_decode(np.arange(127)).astype(np.float64)
    assert np.all(np.diff(v) > 0)
    # normal range: 8 values per binade, ratio 2 between bytes 8 apart
    assert np.allclose(v[16:127] / v[8:119], 2.0)
    assert np.all(np.isnan(orc.ue4m3_decode([0x7F])))


def test_ue4m3_matches_torch_float8(orc):
    # torch's float8_e4m3fn cast is round-to-nearest-even; agrees on [0, 448].
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(-12, 6, 20000)),
                        orc.ue4m3_decode(np.arange(127)).astype(np.float64)]).astype(np.float32)
    v = v[v <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(orc.ue4m3_encode(v), ref)
    assert orc.ue4m3_encode([1000.0])[0] == 0x7E and orc.ue4m3_encode([0.0])[0] == 0


# ------------------------------------------------------- 16-bit rounding

def test_half_conversions_match_numpy_and_torch(orc):
    rng = np.random.default_rng(3)
    h = rng.integers(0, 65536, 4000).astype(np.uint16)
    h = h[(h & 0x7C00) != 0x7C00]
    assert np.array_equal(orc.half_to_float(h, 0), h.view(np.float16).astype(np.float32))
    b = rng.integers(0, 65536, 4000).astype(np.uint16)
    b = b[(b & 0x7F80) != 0x7F80]
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float().numpy()
    assert np.array_equal(orc.half_to_float(b, 1), ref)
    x = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e-6, 500)])
    assert np.array_equal(orc.double_to_half(x, 0), x.astype(np.float16).view(np.uint16))
    xf = x.astype(np.float32).astype(np.float64)  # exactly representable in fp32
    refb = torch.from_numpy(xf.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(orc.double_to_half(xf, 1), refb.view(np.uint16))


# -------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("d", [16, 64, 128])
def test_fwht_is_sylvester_hadamard(orc, d):
    from scipy.linalg import hadamard
    Hm = hadamard(d).astype(np.float64)
    # H H^T = d I through the transform of the identity rows
    assert np.array_equal(orc.fwht_rows(np.eye(d, dtype=np.float32)), Hm.astype(np.float32))
    rng = np.random.default_rng(d)
    x = rng.integers(-8, 9, (7, d)).astype(np.float32)  # exact in fp32
    assert np.array_equal(orc.fwht_rows(x).astype(np.float64), x.astype(np.float64) @ Hm.T)


def test_fwht_preserves_scores(orc):
    # ScaleSearchAttention: the rotation keeps the attention scores.
    rng = np.random.default_rng(5)
    q = rng.integers(-4, 5, (9, 128)).astype(np.float32)
    k = rng.integers(-4, 5, (11, 128)).astype(np.float32)
    qh, kh = orc.fwht_rows(q).astype(np.float64), orc.fwht_rows(k).astype(np.float64)
    assert np.array_equal(qh @ kh.T / 128.0, q.astype(np.float64) @ k.T.astype(np.float64))


# ------------------------------------------------------------ quantiser

def test_max_scaling_maps_absmax_to_six(orc):
    # ScaleSearch page, "Mecanismo" / "Fundamento": offset 0 maps the largest
    # magnitude of the block to the FP4 value 6.
    x = synth.randn16((512, 128), torch.float16, 7)
    codes, scales, g, f = orc.nvfp4_quantize(synth.as_u16(x), 0, use_ss=False)
    assert np.all(f == 0)
    xf = x.float().numpy().reshape(512, 8, 16)
    arg = np.argmax(np.abs(xf), axis=2)
    c = np.stack([codes & 0xF, codes >> 4], -1).reshape(512, 8, 16)
    top = np.take_along_axis(c, arg[..., None], 2)[..., 0]
    normal = scales >= 8
    assert normal.mean() > 0.99
    assert np.all((top[normal] & 7) == 7)


def test_exact_grid_block_is_lossless(orc):
    # A block whose values are E2M1 grid points times a UE4M3 scale times g
    # quantises exactly (dequantised == input).
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    rng = np.random.default_rng(8)
    vals = grid[rng.integers(0, 8, (64, 16))] * np.where(rng.random((64, 16)) < .5, -1, 1)
    vals[:, 0] = 6.0
    # absmax 6 * 0.4375 = 2.625 = 2688 * 2^-10: g = 2^-10 and S = 448 exactly
    x = (vals * 0.4375).astype(np.float16)
    codes, scales, g, _ = orc.nvfp4_quantize(x.view(np.uint16), 0)
    deq = orc.dequantize(codes, scales, g)
    assert np.array_equal(deq.reshape(64, 16), x.astype(np.float64))


def test_scalesearch_never_worse_than_max_scaling(orc):
    x = synth.randn16((2048, 128), torch.float16, 9)
    xf = x.float().numpy().reshape(-1, 16)
    _, s0, g, _ = orc.nvfp4_quantize(synth.as_u16(x), 0, use_ss=False)
    _, s1, g1, f = orc.nvfp4_quantize(synth.as_u16(x), 0, use_ss=True)
    assert g == g1
    s0, s1 = s0.reshape(-1), s1.reshape(-1)
    assert np.array_equal(s1, (s0.astype(int) + f.reshape(-1)).astype(np.uint8))
    e0 = np.array([orc.block_err(xf[i], g, s0[i]) for i in range(0, len(s0), 7)])
    e1 = np.array([orc.block_err(xf[i], g, s1[i]) for i in range(0, len(s1), 7)])
    assert np.all(e1 <= e0)
    assert np.mean(e1) < 0.9 * np.mean(e0)


def _orig_domain_err(x, g, S, grid_vals):
    """Squared error in the input domain of the nearest-grid quantisation of x
    with block scale value S (independent numpy restatement of dequantise)."""
    dec = np.float64(S) * np.float64(g)
    t = x.astype(np.float64) / dec
    q = grid_vals[np.argmin(np.abs(t[:, None] - grid_vals[None, :]), axis=1)]
    return float(np.sum((x.astype(np.float64) - q * dec) ** 2))


def test_scalesearch_brute_force_window(orc):
    # ScaleSearch page, "Estrategia de Busqueda": exhaustive search over the
    # offsets f in [-2, 6] for the scale of least block MSE.
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6], np.float64)
    rng = np.random.default_rng(10)
    g = np.float32(1.0 / 2688.0 * 8.0)
    for trial in range(300):
        x = (rng.normal(0, 1, 16) * rng.choice([0.05, 1.0, 3.0])).astype(np.float32)
        _, S0, f0 = orc.quant_block(x, g, False)
        _, S, f = orc.quant_block(x, g, True)
        assert f0 == 0 and S == S0 + f and -2 <= f <= 6
        sv = orc.ue4m3_decode(np.arange(127)).astype(np.float64)
        errs = {ff: _orig_domain_err(x, g, sv[S0 + ff], grid)
                for ff in range(-2, 7) if 1 <= S0 + ff <= 126}
        best = min(errs.values())
        assert errs[f] <= best * (1 + 1e-5) + 1e-30, (trial, f, errs)


def test_scalesearch_bimodal_offsets(orc):
    # ScaleSearch page, "Fundamento": on Gaussian data the best offsets are
    # bimodal -- a mode at 0 and a second one where the block absmax maps to
    # FP4 4, a scale about 1.5x larger.
    x = synth.randn16((4096, 128), torch.float16, 11)
    _, s, g, f = orc.nvfp4_quantize(synth.as_u16(x), 0, use_ss=True)
    hist = np.bincount(f.reshape(-1) + 2, minlength=9)
    assert np.argmax(hist) == 2  # f = 0
    pos = hist[3:]
    fmode = int(np.argmax(pos)) + 1
    assert pos[fmode - 1] > 0.5 * hist[2]
    s0 = s.reshape(-1).astype(int) - f.reshape(-1)
    sel = (f.reshape(-1) == fmode) & (s0 >= 8)
    ratio = orc.ue4m3_decode(s.reshape(-1)[sel]) / orc.ue4m3_decode(s0[sel].astype(np.uint8))
    assert 1.3 < float(np.median(ratio)) < 1.7
    # a dip between the modes
    assert hist[2 + 2] < 0.5 * min(hist[2], pos[fmode - 1])


def test_tensor_scale_and_power_of_two_invariance(orc):
    x = synth.randn16((256, 64), torch.float16, 12)
    c1, s1, g1, _ = orc.nvfp4_quantize(synth.as_u16(x), 0, use_ss=True)
    assert g1 == np.float32(np.abs(x.float().numpy()).max()) / np.float32(2688)
    c2, s2, g2, _ = orc.nvfp4_quantize(synth.as_u16((x.float() * 4).half()), 0, use_ss=True)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    z = np.zeros((16, 32), np.uint16)
    c, s, g, _ = orc.nvfp4_quantize(z, 0)
    assert g == 1.0 and not c.any() and not s.any()


def test_colblocks_is_transposed_rowblocks(orc):
    x = synth.randn16((64, 48), torch.bfloat16, 13)
    c, s, g, f = orc.nvfp4_quantize_colblocks(synth.as_u16(x), 1, use_ss=True)
    ct, st, gt, ft = orc.nvfp4_quantize(synth.as_u16(x.t().contiguous()), 1, use_ss=True)
    assert g == gt and np.array_equal(c, ct) and np.array_equal(s, st) and np.array_equal(f, ft)


# ------------------------------------------------------------- selection

def test_topk_counts_golden(orc):
    for frac, n, k in _table("topk_counts.txt"):
        assert orc.topk_count(np.float32(float(frac)), int(n)) == int(k)


@pytest.mark.parametrize("causal", [False, True])
def test_selection_brute_force(orc, causal):
    B, N, H, Hkv, d, blk = 2, 200, 4, 2, 32, 32
    q = synth.randn16((B, N, H, d), torch.bfloat16, 20)
    k = synth.randn16((B, N, Hkv, d), torch.bfloat16, 21)
    mask, scores = orc.block_mean_topk(synth.as_u16(q), synth.as_u16(k), 1, blk, causal, 0.3)
    nb = (N + blk - 1) // blk
    qf, kf = q.double().numpy(), k.double().numpy()
    for b in range(B):
        for h in range(H):
            qm = np.stack([qf[b, i * blk:(i + 1) * blk, h].mean(0) for i in range(nb)])
            km = np.stack([kf[b, j * blk:(j + 1) * blk, h // (H // Hkv)].mean(0) for j in range(nb)])
            sc = qm @ km.T
            assert np.allclose(scores[b, h], sc, rtol=1e-12, atol=1e-13)
            valid = [(i, j) for i in range(nb) for j in range(nb) if not causal or j <= i]
            kk = math.ceil(np.float64(np.float32(0.3)) * len(valid) - 1e-9)
            order = sorted(valid, key=lambda ij: (-sc[ij], ij[0] * nb + ij[1]))
            want = np.zeros((nb, nb), np.uint8)
            for ij in order[:kk]:
                want[ij] = 1
            assert np.array_equal(mask[b, h], want)


@pytest.mark.parametrize("causal", [False, True])
def test_sink_blocks_are_added_to_topk(orc, causal):
    # ScaleSearchAttention, sink-aware mixed precision: the first and the
    # most recent key blocks stay at full precision.  Brute force over the
    # pairs: the selection is the top-k set (quota unchanged) united with
    # the fixed pairs, and nothing outside the valid pairs.
    B, N, H, Hkv, d, blk = 1, 300, 3, 1, 32, 32
    q = synth.randn16((B, N, H, d), torch.bfloat16, 30)
    k = synth.randn16((B, N, Hkv, d), torch.bfloat16, 31)
    nb = (N + blk - 1) // blk
    for frac, sink, recent in [(0.0, 1, 1), (0.2, 1, 2), (0.3, 2, 0), (0.1, 0, 3), (0.0, 20, 0)]:
        base, _ = orc.block_mean_topk(synth.as_u16(q), synth.as_u16(k), 1, blk, causal, frac)
        mask, _ = orc.block_mean_topk(synth.as_u16(q), synth.as_u16(k), 1, blk, causal, frac,
                                      sink_blocks=sink, recent_blocks=recent)
        for h in range(H):
            for i in range(nb):
                seen = [j for j in range(nb) if not causal or j <= i]
                newest = seen[-recent:] if recent else []
                for j in range(nb):
                    fixed = j in seen and (j < sink or j in newest)
                    want = 1 if (base[0, h, i, j] or fixed) else 0
                    assert mask[0, h, i, j] == want, (frac, sink, recent, h, i, j)
        if sink >= nb:  # every valid pair
            valid = nb * (nb + 1) // 2 if causal else nb * nb
            assert mask.sum() == H * valid


def test_selection_ties_go_to_lower_index(orc):
    q = torch.ones((1, 128, 1, 16), dtype=torch.float16)
    k = torch.ones((1, 128, 1, 16), dtype=torch.float16)
    mask, _ = orc.block_mean_topk(synth.as_u16(q), synth.as_u16(k), 0, 16, False, 0.25)
    flat = mask.reshape(-1)
    assert flat[:16].all() and not flat[16:].any()


def test_selection_varlen_matches_per_sequence(orc):
    lens = [70, 33, 128]
    cu = np.array([0, 70, 103, 231], np.int32)
    q = synth.randn16((231, 2, 16), torch.float16, 22)
    k = synth.randn16((231, 1, 16), torch.float16, 23)
    m = orc.block_mean_topk_varlen(synth.as_u16(q), synth.as_u16(k), 0, cu, 32, True, 0.4)
    off = 0
    for s, L in enumerate(lens):
        ms, _ = orc.block_mean_topk(synth.as_u16(q[cu[s]:cu[s + 1]][None]),
                                    synth.as_u16(k[cu[s]:cu[s + 1]][None]), 0, 32, True, 0.4)
        assert np.array_equal(m[off:off + ms.size], ms.reshape(-1))
        off += ms.size
    assert off == m.size
