"""Pins of the oracle's Attn-QAT backward (reading R17; "Attn-QAT",
Metodologia, items 1 and 2) against torch fp64 autograd of the same fake-quantised
graph with straight-through quantisers, an implementation of the gradient
independent of the oracle's.  Autograd takes the softmax gradient's row
scalar as rowsum(P o dP) = dO . (P V^), i.e. from the high-precision output
O' the pages prescribe; the FP4 output O = P^ V^ in its place gives other
gradients (also checked)."""
import numpy as np
import pytest
import torch

BF16 = 1


def _bf16(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _f32(h):
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _deq_rows(orc, x16, d):
    codes, scales, g, _ = orc.nvfp4_quantize(x16.reshape(-1, d), BF16)
    return orc.dequantize(codes, scales, g).reshape(x16.shape)


def _deq_v(orc, v16, L, Hkv, d):
    # 16-blocks along the tokens (L a multiple of 16 here)
    codes, scales, g, _ = orc.nvfp4_quantize_colblocks(v16.reshape(L, Hkv * d), BF16)
    return orc.dequantize(codes, scales, g).T.reshape(L, Hkv, d)


def _p_hat(orc, P, blk):
    """Two-level FP4 image of normalised probability rows per key tile."""
    L = P.shape[-1]
    out = np.zeros_like(P)
    for idx in np.ndindex(P.shape[:-1]):
        row = P[idx].astype(np.float32)
        for j0 in range(0, L, blk):
            pt = row[j0:j0 + blk]
            rm = np.float32(pt.max())
            if rm == 0:
                continue
            ph = pt * (np.float32(2688.0) / rm)
            sigma = rm / np.float32(2688.0)
            for b0 in range(0, len(ph), 16):
                blkv = ph[b0:b0 + 16]
                S = orc.ue4m3_encode(np.array([blkv.max() / np.float32(6.0)], np.float32))[0]
                dec = np.float32(orc.ue4m3_decode([S])[0])
                if S == 0:
                    continue
                codes = orc.e2m1_encode(blkv * (np.float32(1.0) / dec))
                out[idx][j0 + b0:j0 + b0 + len(blkv)] = (
                    orc.e2m1_decode(codes).astype(np.float64) * float(dec) * float(sigma))
    return out


@pytest.mark.parametrize("causal,H,Hkv", [(False, 2, 2), (True, 2, 1)])
def test_gradients_match_autograd_with_straight_through(orc, causal, H, Hkv):
    rng = np.random.default_rng(5)
    L, d, blk = 96, 32, 32
    q16 = _bf16(rng.standard_normal((L, H, d)))
    k16 = _bf16(rng.standard_normal((L, Hkv, d)) + 2.0 * rng.standard_normal((1, Hkv, d)))
    v16 = _bf16(rng.standard_normal((L, Hkv, d)))
    do16 = _bf16(rng.standard_normal((L, H, d)))
    cu = np.array([0, L], np.int32)
    r = orc.attn_qat_bwd(q16, k16, v16, do16, BF16, cu, blk, causal)

    qh = torch.tensor(_deq_rows(orc, q16, d), dtype=torch.float64)
    kh = torch.tensor(_deq_rows(orc, k16, d), dtype=torch.float64)
    vh = torch.tensor(_deq_v(orc, v16, L, Hkv, d), dtype=torch.float64)
    q = torch.tensor(_f32(q16), dtype=torch.float64, requires_grad=True)
    k = torch.tensor(_f32(k16), dtype=torch.float64, requires_grad=True)
    v = torch.tensor(_f32(v16), dtype=torch.float64, requires_grad=True)
    dO = torch.tensor(_f32(do16), dtype=torch.float64)
    # straight-through fake quantisers
    Qs = q + (qh - q).detach()
    Ks = k + (kh - k).detach()
    Vs = v + (vh - v).detach()
    g = H // Hkv
    Kx = Ks.repeat_interleave(g, dim=1)
    Vx = Vs.repeat_interleave(g, dim=1)
    S = torch.einsum("ihc,jhc->hij", Qs, Kx) / np.sqrt(d)
    if causal:
        S = S.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    P = torch.softmax(S, dim=-1)
    Ph = torch.tensor(_p_hat(orc, P.detach().numpy(), blk))
    Pst = P + (Ph - P).detach()
    O = torch.einsum("hij,jhc->ihc", Pst, Vx)
    (O * dO).sum().backward()

    np.testing.assert_allclose(r["o"], O.detach().numpy(), rtol=0, atol=1e-12)
    o_hp = torch.einsum("hij,jhc->ihc", P, Vx).detach().numpy()
    np.testing.assert_allclose(r["o_hp"], o_hp, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], torch.logsumexp(S, -1).detach().numpy(), rtol=0, atol=1e-12)
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        want = t.grad.numpy()
        np.testing.assert_allclose(r[name], want, rtol=0, atol=1e-10 * max(1.0, np.abs(want).max()))

    # the FP4 output in place of O' gives other gradients
    Dn = (O.detach() * dO).sum(-1)                       # [i, h]
    dP = torch.einsum("ihc,jhc->hij", dO, Vx.detach())
    dS = P.detach() * (dP - Dn.T[:, :, None])
    dq_naive = torch.einsum("hij,jhc->ihc", dS, Kx.detach()) / np.sqrt(d)
    assert np.abs(dq_naive.numpy() - r["dq"]).max() > 1e-4 * np.abs(r["dq"]).max()


@pytest.mark.parametrize("causal", [False, True])
def test_p_hat_structure_through_identity_values(orc, causal):
    """With V the identity (d = L), V^ = v I, so the oracle's outputs expose
    the probabilities row by row: O' = v P and O = v P^.  Closed-form
    properties of the two-level quantisation (reading R7 on the normalised
    rows): on each key tile sigma = max P / 2688; each 16-key block of P^ is
    (an E2M1 value) x (one UE4M3 value) x sigma; the tile maximum is
    reproduced exactly (2688 / 6 = 448, the largest UE4M3 value, with code
    6); and no element moves by more than one grid unit (the gap 4 -> 6 is
    the widest) times its block's scale."""
    rng = np.random.default_rng(11)
    L, blk = 64, 32
    q16 = _bf16(rng.standard_normal((L, 1, L)))
    k16 = _bf16(rng.standard_normal((L, 1, L)))
    v16 = _bf16(np.eye(L).reshape(L, 1, L))
    do16 = _bf16(rng.standard_normal((L, 1, L)))
    r = orc.attn_qat_bwd(q16, k16, v16, do16, BF16, np.array([0, L], np.int32), blk, causal)
    vhat = _deq_v(orc, v16, L, 1, L)[:, 0, :]
    vv = vhat[0, 0]
    assert np.array_equal(vhat, vv * np.eye(L))  # one value on the diagonal
    P = r["o_hp"][:, 0, :] / vv
    Ph = r["o"][:, 0, :] / vv
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    scales = np.array([orc.ue4m3_decode([b])[0] for b in range(1, 127)], np.float64)
    for i in range(L):
        kend = i + 1 if causal else L
        assert np.all(P[i, kend:] == 0) and np.all(Ph[i, kend:] == 0)
        for j0 in range(0, kend, blk):
            p, ph = P[i, j0:min(kend, j0 + blk)], Ph[i, j0:min(kend, j0 + blk)]
            m = p.max()
            sigma = float(np.float32(np.float32(m) / np.float32(2688.0)))
            jm = int(np.argmax(p))
            assert abs(ph[jm] - m) <= 4e-7 * m, (i, j0)
            for b0 in range(0, len(p), 16):
                blkv = ph[b0:b0 + 16] / sigma
                if not blkv.any():
                    continue
                # one UE4M3 scale puts every element on the E2M1 grid
                ok = [s for s in scales
                      if np.all(np.min(np.abs(blkv[:, None] / s - grid[None, :]), axis=1) <= 1e-5)]
                assert ok, (i, j0, b0)
                s = min(ok, key=lambda x: abs(blkv.max() / x - 6))
                # max scaling: the block maximum carries code 6 (normal scales)
                if s >= 2.0 ** -6:
                    assert abs(blkv.max() / s - 6.0) <= 1e-5, (i, j0, b0)
                assert np.all(np.abs(ph[b0:b0 + 16] - p[b0:b0 + 16]) <= (1.0 + 1e-5) * s * sigma)
