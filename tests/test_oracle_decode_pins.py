"""Pins the oracle's decode step (one query token per sequence against the
FP4 + FP16 double cache; ThriftAttention, Resultados and Significado) to
facts other than itself: the prefill oracle's last query row (an independent
implementation of the same per-row steps), unquantised fp64 attention within
the 16-bit rounding of P, closed forms for a one-token cache, and a brute-force
selection with exactly rounded fused multiply-adds."""
import math
from fractions import Fraction

import numpy as np
import pytest

BF16 = 1


def _bf16(x):
    """float32 array -> bf16 bit patterns (round to nearest even)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _f32(h):
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _cache(rng, B, ncap, Hkv, d, scale=1.0):
    k = _bf16(rng.standard_normal((B, ncap, Hkv, d)) * scale + 0.5 * rng.standard_normal(d))
    v = _bf16(rng.standard_normal((B, ncap, Hkv, d)))
    return k, v


def _prefill_last_rows(orc, q, k, v, lens, blk, dmask, sink=0, recent=0):
    """Prefill oracle, causal, on sequences whose every query row is the
    decode query; returns (out64 [B,H,d], lse [B,H], tol, (gq, gk, gv))."""
    B, H, d = q.shape
    Hkv = k.shape[2]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Q = np.concatenate([np.broadcast_to(q[b], (lens[b], H, d)) for b in range(B)])
    K = np.concatenate([k[b, :lens[b]] for b in range(B)])
    V = np.concatenate([v[b, :lens[b]] for b in range(B)])
    masks, units = [], []
    for b in range(B):
        nb = (lens[b] + blk - 1) // blk
        m = np.zeros((H, nb, nb), np.uint8)
        m[:, nb - 1, :] = dmask[b, :, :nb]
        masks.append(m.reshape(-1))
        for h in range(H):
            units.append((b, h, nb - 1))
    r = orc.thrift_attn(Q, K, V, BF16, cu, blk, True, 0.0, mask=np.concatenate(masks),
                        units=np.array(units, np.int32))
    last = cu[1:] - 1
    return r["out64"][last], r["lse"][:, last].T, r["tol"][last], r["g"]


@pytest.mark.parametrize("frac,sink,recent", [(0.0, 0, 0), (0.3, 0, 0), (0.5, 1, 1), (1.0, 0, 0)])
def test_decode_equals_prefill_last_row(orc, frac, sink, recent):
    rng = np.random.default_rng(11)
    B, H, Hkv, d, blk, ncap = 3, 4, 2, 64, 64, 320
    lens = np.array([300, 64, 129], np.int32)
    k, v = _cache(rng, B, ncap, Hkv, d)
    q = _bf16(rng.standard_normal((B, H, d)) * 1.5)
    # the prefill derives g_K, g_V from the real tokens; the cache is given them
    K = np.concatenate([k[b, :lens[b]] for b in range(B)])
    V = np.concatenate([v[b, :lens[b]] for b in range(B)])
    g_kv = (orc.tensor_scale(K.reshape(-1, d), BF16), orc.tensor_scale(V.reshape(-1, d), BF16))
    dec = orc.thrift_decode(q, k, v, BF16, lens, blk, g_kv, frac, sink_blocks=sink,
                            recent_blocks=recent)
    again = orc.thrift_decode(q, k, v, BF16, lens, blk, g_kv, frac, sink_blocks=sink,
                              recent_blocks=recent, gq=dec["gq"])
    assert np.array_equal(again["out64"], dec["out64"])  # g_Q given = g_Q derived
    o64, lse, tol, g = _prefill_last_rows(orc, q, k, v, lens, blk, dec["mask"])
    assert g[1] == g_kv[0] and g[2] == g_kv[1] and g[0] == dec["gq"]
    assert np.array_equal(dec["out64"], o64)
    assert np.array_equal(dec["lse"], lse)
    assert np.array_equal(dec["tol"], tol)
    nfp16 = dec["mask"].sum()
    if frac == 0.0 and sink == 0:
        assert nfp16 == 0
    if frac == 1.0:
        assert nfp16 == sum(H * ((L + blk - 1) // blk) for L in lens)


def test_decode_all_fp16_is_softmax_within_p_rounding(orc):
    rng = np.random.default_rng(5)
    B, H, Hkv, d, blk, ncap = 2, 4, 4, 64, 64, 256
    lens = np.array([256, 77], np.int32)
    k, v = _cache(rng, B, ncap, Hkv, d)
    q = _bf16(rng.standard_normal((B, H, d)))
    dec = orc.thrift_decode(q, k, v, BF16, lens, blk, (1.0, 1.0), 1.0)
    cu = np.array([0, lens[0], lens[0] + lens[1]], np.int32)
    K = np.concatenate([k[b, :lens[b]] for b in range(B)])
    V = np.concatenate([v[b, :lens[b]] for b in range(B)])
    # fp64 attention of the query as the last token of each sequence
    Q = np.zeros((cu[-1], H, d), np.uint16)
    for b in range(B):
        Q[cu[b + 1] - 1] = q[b]
    rows = np.array([(cu[b + 1] - 1, h) for b in range(B) for h in range(H)], np.int64)
    ref, lse = orc.attn_fp64(Q, K, V, BF16, cu, True, rows=rows)
    vmax = np.abs(_f32(v)).max()
    for b in range(B):
        got = dec["out64"][b]
        want = ref[cu[b + 1] - 1]
        # P rounded to bf16: |dP| <= 2^-9 P, so |dO| <= 2^-9 max|v|
        assert np.abs(got - want).max() <= 2.0 ** -9 * vmax * 1.0001
        # l sums the unrounded probabilities: lse agrees to fp32 rounding
        np.testing.assert_allclose(dec["lse"][b], lse[:, cu[b + 1] - 1], rtol=0, atol=2e-6)


def test_decode_one_token_closed_forms(orc):
    """A one-token cache: P = [1].  FP16: out = v0 and lse = q.k / sqrt(d).
    NVFP4: Phat = 2688 sits on the grid exactly (E2M1 6 x UE4M3 448), so out
    is v0 quantised as a V block of sixteen tokens with fifteen zeros,
    dequantised (the block quantiser is pinned on its own), up to the fp32
    rounding of sigma = 1/2688."""
    rng = np.random.default_rng(3)
    B, H, Hkv, d, blk, ncap = 2, 2, 1, 32, 16, 16
    lens = np.array([1, 1], np.int32)
    k, v = _cache(rng, B, ncap, Hkv, d)
    q = _bf16(rng.standard_normal((B, H, d)))
    gv = 0.0123
    full = orc.thrift_decode(q, k, v, BF16, lens, blk, (0.01, gv), 1.0)
    for b in range(B):
        for h in range(H):
            assert np.array_equal(full["out64"][b, h], _f32(v[b, 0, 0]).astype(np.float64))
            s = np.dot(_f32(q[b, h]).astype(np.float64), _f32(k[b, 0, 0]).astype(np.float64))
            assert abs(full["lse"][b, h] - s / math.sqrt(d)) <= 1e-6 * max(1.0, abs(s))
    fp4 = orc.thrift_decode(q, k, v, BF16, lens, blk, (0.01, gv), 0.0)
    for b in range(B):
        v0 = _f32(v[b, 0, 0])
        want = np.zeros(d)
        for c in range(d):
            col = np.zeros(16, np.float32)
            col[0] = v0[c]
            codes, S, _ = orc.quant_block(col, gv, False)
            want[c] = (float(orc.e2m1_decode([codes[0] & 15])[0]) * float(orc.ue4m3_decode([S])[0])
                       * float(np.float32(gv)))
        for h in range(H):
            # exact up to the fp32 rounding of sigma = 1/2688 (reading R7)
            np.testing.assert_allclose(fp4["out64"][b, h], want, rtol=2.0 ** -23, atol=0)


def _fma(a, b, c):
    return float(Fraction(a) * Fraction(b) + Fraction(c))


@pytest.mark.parametrize("frac,sink,recent", [(0.25, 0, 0), (0.5, 1, 2), (0.0, 2, 0), (1.0, 0, 0)])
def test_decode_selection_brute_force(orc, frac, sink, recent):
    rng = np.random.default_rng(21)
    B, H, Hkv, d, blk, ncap = 3, 4, 2, 16, 16, 120
    lens = np.array([120, 37, 16], np.int32)
    k, v = _cache(rng, B, ncap, Hkv, d)
    # two identical key blocks in sequence 0: equal scores, ties to lower j
    k[0, 32:48] = k[0, 64:80]
    q = _bf16(rng.standard_normal((B, H, d)))
    r = orc.thrift_decode(q, k, v, BF16, lens, blk, (0.01, 0.01), frac, sink_blocks=sink,
                          recent_blocks=recent)
    nbcap = (ncap + blk - 1) // blk
    kf = _f32(k.reshape(-1)).reshape(k.shape)
    for b in range(B):
        nb = (lens[b] + blk - 1) // blk
        for h in range(H):
            hk = h // (H // Hkv)
            qb = [float(x) for x in _f32(q[b, h])]
            sc = []
            for j in range(nb):
                t0, t1 = j * blk, min(lens[b], j * blk + blk)
                km = []
                for c in range(d):
                    acc = 0.0
                    for t in range(t0, t1):
                        acc += float(kf[b, t, hk, c])
                    km.append(acc / (t1 - t0))
                acc = 0.0
                for c in range(d):
                    acc = _fma(qb[c], km[c], acc)
                sc.append((acc, j))
            kk = min(nb, max(0, math.ceil(frac * nb - 1e-9)))
            order = sorted(sc, key=lambda x: (-x[0], x[1]))
            want = np.zeros(nbcap, np.uint8)
            for _, j in order[:kk]:
                want[j] = 1
            for j in range(nb):
                if j < sink or j >= nb - recent:
                    want[j] = 1
            assert np.array_equal(r["mask"][b, h], want), (b, h)


def test_decode_empty_sequence(orc):
    rng = np.random.default_rng(1)
    k, v = _cache(rng, 2, 32, 1, 16)
    q = _bf16(rng.standard_normal((2, 2, 16)))
    r = orc.thrift_decode(q, k, v, BF16, np.array([0, 5], np.int32), 16, (0.01, 0.01), 0.5)
    assert np.all(r["out"][0] == 0) and np.all(np.isneginf(r["lse"][0]))
    assert np.all(r["mask"][0] == 0) and np.all(np.isfinite(r["lse"][1]))
