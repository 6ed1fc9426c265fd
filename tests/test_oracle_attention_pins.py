"""Pins the oracle's attention emulation and its fp64 reference.

Closed forms (uniform scores, one-hot rows), library routines (torch SDPA in
float64), special cases (all pairs FP16 reduces to 16-bit attention), the
quality trend the ThriftAttention page reports (more FP16 pairs, less error),
and invariants (tiling, sampling of units).
"""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import synth


def _packed(B, N, H, Hkv, d, dtype, seed, k_off=0.0):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn((B * N, H, d), generator=gen).to(dtype)
    k = (torch.randn((B * N, Hkv, d), generator=gen) + k_off).to(dtype)
    v = torch.randn((B * N, Hkv, d), generator=gen).to(dtype)
    cu = np.arange(B + 1, dtype=np.int32) * N
    return q, k, v, cu


def _f(orc, u16, dt):
    return orc.half_to_float(u16, dt).astype(np.float64)


@pytest.mark.parametrize("causal", [False, True])
def test_fp64_reference_matches_torch_sdpa(orc, causal):
    B, N, H, Hkv, d = 2, 40, 4, 2, 16
    q, k, v, cu = _packed(B, N, H, Hkv, d, torch.bfloat16, 1)
    out, lse = orc.attn_fp64(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, causal)
    qt = q.double().view(B, N, H, d).transpose(1, 2)
    kt = k.double().view(B, N, Hkv, d).transpose(1, 2).repeat_interleave(H // Hkv, 1)
    vt = v.double().view(B, N, Hkv, d).transpose(1, 2).repeat_interleave(H // Hkv, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)
    ref = ref.transpose(1, 2).reshape(B * N, H, d).numpy()
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-12)
    s = (qt @ kt.transpose(-1, -2)) / np.sqrt(d)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    lref = torch.logsumexp(s, -1).permute(1, 0, 2).reshape(H, B * N).numpy()
    assert np.allclose(lse, lref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype,dt,tol", [(torch.float16, 0, 2e-3), (torch.bfloat16, 1, 1.6e-2)])
def test_all_pairs_fp16_is_16bit_attention(orc, dtype, dt, tol):
    # ThriftAttention, Metodologia step 2: selected pairs run in FP16; with a
    # budget of every pair the method is plain 16-bit attention.
    q, k, v, cu = _packed(1, 192, 2, 1, 32, dtype, 2)
    r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), dt, cu, 64, True, 1.0)
    assert r["mask"].sum() == 2 * 6  # every causal pair of the 3x3 block grid, 2 heads
    ref, lref = orc.attn_fp64(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), dt, cu, True)
    out = _f(orc, r["out"], dt)
    assert np.max(np.abs(out - ref)) < tol
    assert np.max(np.abs(r["lse"] - lref)) < 1e-5


def _grid_tensor(shape, rng, scale=0.4375):
    """Values on the E2M1 grid times `scale`; every 16-block along axis 0
    (tokens) and along the last axis holds a 6 so block absmax = 6*scale."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    vals = grid[rng.integers(0, 8, shape)] * np.where(rng.random(shape) < .5, -1, 1)
    vals[::16, ...] = 6.0
    vals[..., ::16] = 6.0
    return torch.from_numpy(vals * scale).to(torch.float16)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("frac", [0.0, 0.5])
def test_uniform_scores_closed_form(orc, causal, frac):
    # Q = 0 makes every score 0: P is uniform, so every probability block is
    # exactly representable (scale 448, code 6) and the output is the mean
    # of the visible V rows; lse = ln(#visible keys).
    N, d = 160, 32
    rng = np.random.default_rng(3)
    q = torch.zeros((N, 1, d), dtype=torch.float16)
    k = torch.from_numpy(rng.normal(0, 1, (N, 1, d))).to(torch.float16)
    v = _grid_tensor((N, 1, d), rng)
    cu = np.array([0, N], np.int32)
    r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, 32, causal, frac)
    vf = v.double().numpy()[:, 0]
    cnt = np.arange(1, N + 1) if causal else np.full(N, N)
    want = np.cumsum(vf, 0) / cnt[:, None] if causal else np.repeat(vf.mean(0)[None], N, 0)
    out = _f(orc, r["out"], 0)[:, 0]
    assert np.max(np.abs(out - want)) < 1e-3
    assert np.allclose(r["lse"][0], np.log(cnt), atol=1e-6)


def test_one_hot_rows_pick_one_value(orc):
    # A query that matches one key far better than all others returns that
    # key's value row on either path.
    N, d = 128, 64
    rng = np.random.default_rng(4)
    kf = rng.normal(0, 1, (N, d))
    kf /= np.linalg.norm(kf, axis=1, keepdims=True)
    tgt = rng.permutation(N)
    q = torch.from_numpy(400.0 * kf[tgt])[:, None].to(torch.float16)
    k = torch.from_numpy(kf)[:, None].to(torch.float16)
    v = _grid_tensor((N, 1, d), rng)
    cu = np.array([0, N], np.int32)
    for frac in (0.0, 1.0):
        r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, 32, False,
                            frac)
        out = _f(orc, r["out"], 0)[:, 0]
        want = v.double().numpy()[tgt, 0]
        assert np.max(np.abs(out - want)) < 0.05 * np.abs(want).max()


def test_more_fp16_pairs_less_error(orc):
    # ThriftAttention, Resultados: error falls as the FP16 budget grows
    # (5% -> 10% -> 25%); all pairs in FP16 is the floor.
    errs = {f: [] for f in (0.0, 0.05, 0.25, 1.0)}
    for seed in range(3):
        q, k, v, cu = _packed(1, 512, 2, 2, 64, torch.bfloat16, 10 + seed, k_off=1.0)
        ref, _ = orc.attn_fp64(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, True)
        for f in errs:
            r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, 64,
                                True, f)
            errs[f].append(np.sqrt(np.mean((_f(orc, r["out"], 1) - ref) ** 2)))
    m = [np.mean(errs[f]) for f in (0.0, 0.05, 0.25, 1.0)]
    assert m[0] > m[1] > m[2] > m[3]
    assert m[3] < 0.2 * m[0]


def test_pure_nvfp4_close_to_exact(orc):
    q, k, v, cu = _packed(1, 256, 2, 1, 64, torch.float16, 20)
    ref, _ = orc.attn_fp64(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, False)
    for had in (0, 1):
        r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, 64, False,
                            0.0, use_ss=True, use_had=bool(had))
        out = _f(orc, r["out"], 0)
        cos = np.sum(out * ref) / np.linalg.norm(out) / np.linalg.norm(ref)
        assert cos > 0.98


def test_tiling_invariance_fp16_path(orc):
    # The online softmax merge does not depend on the key tiling.
    q, k, v, cu = _packed(1, 256, 1, 1, 32, torch.float16, 30)
    outs = []
    for blk in (16, 64, 256):
        r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, blk, True,
                            1.0)
        outs.append(_f(orc, r["out"], 0))
    assert np.max(np.abs(outs[0] - outs[2])) < 2e-3
    assert np.max(np.abs(outs[1] - outs[2])) < 2e-3


def test_hadamard_leaves_fp16_path_unchanged(orc):
    q, k, v, cu = _packed(1, 128, 2, 2, 64, torch.float16, 31)
    a = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, 64, False, 1.0)
    b = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 0, cu, 64, False, 1.0,
                        use_had=True)
    assert np.array_equal(a["out"], b["out"])


def test_sampled_units_equal_full_run(orc):
    q, k, v, cu = _packed(2, 96, 2, 1, 32, torch.bfloat16, 32)
    full = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, 32, True,
                           0.2, use_ss=True)
    units = np.array([[0, 1, 2], [1, 0, 0]], np.int32)
    part = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, 32, True,
                           0.2, use_ss=True, units=units)
    for s, h, i in units:
        rows = slice(cu[s] + 32 * i, cu[s] + 32 * (i + 1))
        assert np.array_equal(part["out"][rows, h], full["out"][rows, h])
        assert np.array_equal(part["lse"][h, rows], full["lse"][h, rows])


@pytest.mark.parametrize("causal", [False, True])
def test_nvfp4_probability_structure_through_identity_values(orc, causal):
    """Two-level P quantisation (reading C8) seen through V = the identity
    (d = N, every pair on the NVFP4 path): V^ is one value v on the diagonal,
    so output column j of a row is v x (its FP4 probability) x a factor that
    is constant over a key tile (sigma, the running-max rescale, 1 / l).  On
    each key tile, 2688 x O_ij / O_i,argmax is then (an E2M1 value) x (one
    UE4M3 value per 16-key block) -- the tile maximum maps to 2688 / 6 = 448
    with code 6, as does every block maximum under a normal scale (max
    scaling) -- and lies within one grid unit of the block scale from
    2688 exp(S_ij - max_tile S), S the scores of the quantised Q and K."""
    N, d, blk = 64, 64, 32
    gen = torch.Generator().manual_seed(21)
    q = torch.randn((N, 1, d), generator=gen).to(torch.bfloat16)
    k = torch.randn((N, 1, d), generator=gen).to(torch.bfloat16)
    v = torch.eye(N).reshape(N, 1, N).to(torch.bfloat16)
    cu = np.array([0, N], np.int32)
    r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, blk, causal, 0.0)
    O = r["out64"][:, 0, :]

    def deq(x):
        codes, scales, g, _ = orc.nvfp4_quantize(synth.as_u16(x).reshape(N, d), 1)
        return orc.dequantize(codes, scales, g).astype(np.float64)

    S = deq(q) @ deq(k).T / np.sqrt(d)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    scales = np.array([orc.ue4m3_decode([b])[0] for b in range(1, 127)], np.float64)
    for i in range(N):
        kend = i + 1 if causal else N
        assert np.all(O[i, kend:] == 0)
        for j0 in range(0, kend, blk):
            j1 = min(kend, j0 + blk)
            o, s = O[i, j0:j1], S[i, j0:j1]
            jm = int(np.argmax(s))
            assert o[jm] > 0 and o[jm] == o.max(), (i, j0)
            rq = 2688.0 * o / o[jm]
            exact = 2688.0 * np.exp(s - s[jm])
            for b0 in range(0, j1 - j0, 16):
                blkv = rq[b0:b0 + 16]
                if not blkv.any():
                    continue
                ok = [t for t in scales
                      if np.all(np.min(np.abs(blkv[:, None] / t - grid[None, :]), axis=1) <= 1e-6)]
                assert ok, (i, j0, b0)
                t = min(ok, key=lambda x: abs(blkv.max() / x - 6))
                # max scaling: the block maximum carries code 6 (a normal
                # UE4M3 scale rounds amax / 6 within 2^-4, so amax / S is in
                # [5.65, 6.4] and rounds to 6)
                if t >= 2.0 ** -6:
                    assert abs(blkv.max() / t - 6.0) <= 1e-9, (i, j0, b0)
                assert np.all(np.abs(blkv - exact[b0:b0 + 16]) <= (1.0 + 1e-4) * t), (i, j0, b0)
