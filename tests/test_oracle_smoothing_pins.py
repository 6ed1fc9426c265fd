"""Pins of the oracle's K smoothing (reading R16: NVFP4 path on K - mu with
mu added back to the dequantised keys; FP16 path and selection on raw K)
against facts other than itself: no-op cases that must be bit-identical,
translation invariance of the NVFP4 path, and the accuracy the reading is
for (the mixed path only agrees with fp64 attention if the mean is added back
with the right sign)."""
import numpy as np
import pytest

BF16 = 1


def _bf16(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _f32(h):
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _inputs(seed, lens, H=2, Hkv=1, d=64, offset=0.0):
    rng = np.random.default_rng(seed)
    total = int(sum(lens))
    q = _bf16(rng.standard_normal((total, H, d)))
    k = rng.standard_normal((total, Hkv, d)) + offset * rng.standard_normal((1, Hkv, d))
    v = _bf16(rng.standard_normal((total, Hkv, d)))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return q, _bf16(k), v, cu


def test_channel_means_layout(orc):
    q, k, v, cu = _inputs(0, [300, 77], Hkv=2)
    mu = orc.k_channel_means(k, BF16, cu)
    kf = _f32(k).astype(np.float64)
    for s in range(2):
        rows = kf[cu[s]:cu[s + 1]]
        # block sums of 128 tokens, in order, then in order over blocks
        total = np.zeros(rows.shape[1:])
        for b0 in range(0, len(rows), 128):
            total = total + np.cumsum(rows[b0:b0 + 128], axis=0)[-1]
        assert np.array_equal(mu[s], (total / len(rows)).astype(np.float32))


def test_zero_mean_keys_make_smoothing_a_no_op(orc):
    # tokens in +-pairs: every channel mean is exactly zero
    q, k, v, cu = _inputs(1, [256], H=2, Hkv=2)
    k[1::2] = k[0::2] ^ np.uint16(0x8000)
    assert not orc.k_channel_means(k, BF16, cu).any()
    for frac in (0.0, 0.3):
        a = orc.thrift_attn(q, k, v, BF16, cu, 64, True, frac)
        b = orc.thrift_attn(q, k, v, BF16, cu, 64, True, frac, smooth_k=True)
        assert np.array_equal(a["out64"], b["out64"]) and np.array_equal(a["lse"], b["lse"])


def test_fp16_path_and_selection_ignore_smoothing(orc):
    q, k, v, cu = _inputs(2, [200, 130], offset=4.0)
    a = orc.thrift_attn(q, k, v, BF16, cu, 64, False, 1.0)
    b = orc.thrift_attn(q, k, v, BF16, cu, 64, False, 1.0, smooth_k=True)
    assert np.array_equal(a["out64"], b["out64"])
    c = orc.thrift_attn(q, k, v, BF16, cu, 64, False, 0.25)
    e = orc.thrift_attn(q, k, v, BF16, cu, 64, False, 0.25, smooth_k=True)
    assert np.array_equal(c["mask"], e["mask"])


def test_nvfp4_path_is_translation_invariant(orc):
    # shifting every key of a channel by a constant moves mu by the same
    # constant and leaves K - mu, hence every code, unchanged; the scores of
    # a row all move by q^ . shift, which the softmax removes
    q, k, v, cu = _inputs(3, [192], H=2, Hkv=1)
    k = _bf16(np.round(_f32(k) * 8) / 8)            # multiples of 1/8, |k| < 8
    shift = np.round(np.random.default_rng(9).standard_normal(64) * 4) / 8
    k2 = _bf16(_f32(k) + shift)                     # exact in bf16
    assert np.array_equal(_f32(k2), _f32(k) + shift.astype(np.float32))
    a = orc.thrift_attn(q, k, v, BF16, cu, 64, True, 0.0, smooth_k=True)
    b = orc.thrift_attn(q, k2, v, BF16, cu, 64, True, 0.0, smooth_k=True)
    np.testing.assert_allclose(b["out64"], a["out64"], rtol=0, atol=1e-9)


@pytest.mark.parametrize("frac", [0.25, 0.6])
def test_mixed_paths_see_the_same_scores(orc, frac):
    """K = Kt + mu0 with Kt zero-mean, everything exact in bf16, and q on the
    NVFP4 grid (q^ = q).  Smoothing quantises K - mu = Kt and adds q . mu0 to
    every NVFP4 score; the FP16 path's raw scores carry the same q . mu0.  So
    the output equals the unsmoothed oracle run on Kt with the same FP16
    tiles (every score of a row shifted alike): a wrong sign or a missing
    term puts the two paths out of step."""
    rng = np.random.default_rng(7)
    N, H, d = 384, 2, 64
    e2m1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    qv = e2m1[rng.integers(0, 8, (N, H, d))] * np.where(rng.random((N, H, d)) < 0.5, -1, 1)
    qv[:, :, ::16] = 6.0                      # every 16-block's max is 6 units
    q = _bf16(qv * 0.25)
    kt = np.round(rng.standard_normal((N // 2, 1, d)) * 8) / 8
    kt = np.concatenate([kt, -kt])[rng.permutation(N)]  # exactly zero mean
    # (+-pairs anywhere in the sequence: every block sum and the total are exact)
    mu0 = np.round(rng.standard_normal(d) * 24) / 8
    K = _bf16(kt + mu0)
    Kt = _bf16(kt)
    assert np.array_equal(_f32(K), (kt + mu0).astype(np.float32))
    v = _bf16(rng.standard_normal((N, 1, d)))
    cu = np.array([0, N], np.int32)
    assert np.array_equal(orc.k_channel_means(K, BF16, cu)[0, 0], mu0.astype(np.float32))
    a = orc.thrift_attn(q, K, v, BF16, cu, 64, True, frac, smooth_k=True)
    b = orc.thrift_attn(q, Kt, v, BF16, cu, 64, True, frac, mask=a["mask"])
    assert 0 < a["mask"].sum()
    # equal up to the fp32 rounding of probabilities computed from shifted
    # scores (a path out of step moves outputs by O(1e-1))
    np.testing.assert_allclose(a["out64"], b["out64"], rtol=0, atol=1e-5)


def test_smoothing_recovers_accuracy_under_channel_offsets(orc):
    frac = 0.0
    q, k, v, cu = _inputs(4, [512], H=2, Hkv=1, d=64, offset=20.0)
    # V ramps with the position, so moving weight between the NVFP4 and the
    # FP16 tiles of a row (scores of the two paths out of step) moves the output
    t = np.arange(512, dtype=np.float32)[:, None, None] / 512.0
    sign = np.where(np.arange(64) % 2 == 0, 1.0, -1.0).astype(np.float32)
    v = _bf16(3.0 * t * sign + 0.1 * _f32(v))
    ref, _ = orc.attn_fp64(q, k, v, BF16, cu, True)
    plain = orc.thrift_attn(q, k, v, BF16, cu, 64, True, frac)
    smooth = orc.thrift_attn(q, k, v, BF16, cu, 64, True, frac, smooth_k=True)
    e_plain = np.sqrt(np.mean((plain["out64"] - ref) ** 2))
    e_smooth = np.sqrt(np.mean((smooth["out64"] - ref) ** 2))
    assert e_smooth < 0.5 * e_plain, (e_smooth, e_plain)
