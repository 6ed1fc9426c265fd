"""Decode over the double KV cache (ThriftAttention, Resultados and
Significado) on the GPU against the oracle.

* The cache images the append kernels write are decoded here from the byte
  layout the header documents and compared bit for bit with the oracle's
  quantiser under the same given scales (K rows along d, V in 16-token
  blocks along the tokens from token 0), with the 16-bit tokens themselves,
  and with fp64 sequential block means.
* The decode step against the oracle's decode: selection bit-exact (read
  from the workspace), output within 1e-2 + half a 16-bit ulp + the oracle's
  bound for non-unique roundings, cosine >= 0.9999, lse within 1e-2.
* Shapes: ragged lengths across tile boundaries (1, 129, 1000, ...), an
  empty sequence, G = 1, 4, 8, 16 query heads per kv head, all-NVFP4,
  all-FP16 and mixed selections, sink/recent tiles, fp16 and bf16,
  ScaleSearch, caches filled in several appends, and many splits per
  sequence (small B * Hkv) as well as few.
"""
import dataclasses

import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops, synth

pytestmark = pytest.mark.gpu

from parity_bars import compare


def _compare(got, want64, tol, dtype, what="out"):
    compare(got, want64, dtype, tol, what)


def _gkv(orc, k, v, lengths, dt):
    K = np.concatenate([synth.as_u16(k[b, :L]).reshape(-1, k.shape[-1]) for b, L in
                        enumerate(lengths) if L > 0])
    V = np.concatenate([synth.as_u16(v[b, :L]).reshape(-1, v.shape[-1]) for b, L in
                        enumerate(lengths) if L > 0])
    return (orc.tensor_scale(K, dt), orc.tensor_scale(V, dt))


def _fill(k, v, lengths, capacity, g_kv, dtype, chunks=(1.0,), ss=False):
    """Builds the cache on the GPU by appending each sequence's tokens in
    pieces (fractions of its length, the last piece the remainder)."""
    B, _, Hkv, d = k.shape
    cache = ops.DoubleKVCache(B, Hkv, capacity, g_kv, dtype=dtype, use_scalesearch=ss)
    done = [0] * B
    kc, vc = k.cuda(), v.cuda()
    for ci, frac in enumerate(chunks):
        want = [L if ci == len(chunks) - 1 else min(L, done[b] + int(round(frac * L)))
                for b, L in enumerate(lengths)]
        n_new = [w - d0 for w, d0 in zip(want, done)]
        T = max(1, max(n_new))
        kn = torch.zeros((B, T, Hkv, d), dtype=dtype, device="cuda")
        vn = torch.zeros_like(kn)
        for b in range(B):
            if n_new[b]:
                kn[b, :n_new[b]] = kc[b, done[b]:want[b]]
                vn[b, :n_new[b]] = vc[b, done[b]:want[b]]
        cache.append(kn, vn, torch.tensor(n_new, dtype=torch.int32, device="cuda"))
        done = want
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    assert cache.lengths.cpu().tolist() == list(lengths)
    return cache


# ------------------------------------------------------- the cache images

def _swz(row, byte, pitch):
    chunk = byte >> 4
    sel = (row * pitch >> 7) & (7 if pitch == 128 else 3)
    return row * pitch + ((chunk ^ sel) << 4) + (byte & 15)


def _sf(row, k16):
    return (k16 >> 2) * 512 + (row & 31) * 16 + (row >> 5) * 4 + (k16 & 3)


def _decode_fp4_tile(img, rows=128):
    r = np.arange(rows)[:, None]
    codes = img[_swz(r, np.arange(64)[None, :], 64)]
    scales = img[rows * 64 + _sf(r, np.arange(8)[None, :])]
    return codes, scales


def _decode_f16_tile(img):
    r = np.arange(128)[:, None]
    c = np.arange(128)[None, :]
    off = (c >> 6) * 16384 + _swz(r, (c & 63) * 2, 128)
    return img.view(np.uint8)[off] | (img.view(np.uint8)[off + 1].astype(np.uint16) << 8)


@pytest.mark.parametrize("ss", [False, True])
def test_cache_images_bit_exact(orc, ss):
    w = synth.DecodeWorkload("cache", 2, 4, 2, 512, 0, 0, 128, torch.bfloat16, 0.0, ss)
    lengths = [300, 129]
    inp = synth.make_decode_inputs(w, lengths=lengths)
    k, v = inp["k"], inp["v"]
    g_kv = _gkv(orc, k, v, lengths, 1)
    cache = _fill(k, v, lengths, w.capacity, g_kv, w.dtype, chunks=(0.5, 0.25, 1.0), ss=ss)
    buf = cache.buf.cpu().numpy()
    ntc = (w.capacity + 127) // 128
    ntile = w.B * w.Hkv * ntc
    K4, V4, K16, V16 = 9216, 9216, 32768, 32768
    off = {"k4": 0, "v4": ntile * K4, "k16": ntile * (K4 + V4),
           "v16": ntile * (K4 + V4 + K16)}
    off["mean"] = off["v16"] + ntile * V16
    for b, L in enumerate(lengths):
        nb = (L + 127) // 128
        for hk in range(w.Hkv):
            ku = synth.as_u16(k[b, :L, hk])  # [L, d]
            vu = synth.as_u16(v[b, :L, hk])
            kc, ks, _, _ = orc.nvfp4_quantize(ku, 1, use_ss=ss, g=g_kv[0])
            vpad = np.zeros((nb * 128, 128), np.uint16)
            vpad[:L] = vu
            vc, vs, _, _ = orc.nvfp4_quantize_colblocks(vpad, 1, use_ss=ss, g=g_kv[1])
            for j in range(nb):
                t = (b * w.Hkv + hk) * ntc + j
                n = min(128, L - 128 * j)
                codes, scales = _decode_fp4_tile(buf[off["k4"] + t * K4: off["k4"] + (t + 1) * K4])
                assert np.array_equal(codes[:n], kc[128 * j:128 * j + n]), (b, hk, j)
                assert np.array_equal(scales[:n], ks[128 * j:128 * j + n]), (b, hk, j)
                assert not codes[n:].any() and not scales[n:].any()
                codes, scales = _decode_fp4_tile(buf[off["v4"] + t * V4: off["v4"] + (t + 1) * V4])
                assert np.array_equal(codes, vc[:, 64 * j:64 * j + 64]), (b, hk, j)
                assert np.array_equal(scales, vs[:, 8 * j:8 * j + 8]), (b, hk, j)
                k16 = _decode_f16_tile(buf[off["k16"] + t * K16: off["k16"] + (t + 1) * K16])
                assert np.array_equal(k16[:n], ku[128 * j:128 * j + n])
                assert not k16[n:].any()
                v16 = _decode_f16_tile(buf[off["v16"] + t * V16: off["v16"] + (t + 1) * V16])
                assert np.array_equal(v16[:, :n], vu[128 * j:128 * j + n].T)
                mean = buf[off["mean"] + t * 1024: off["mean"] + (t + 1) * 1024].view(np.float64)
                rows = orc.half_to_float(ku[128 * j:128 * j + n], 1).astype(np.float64)
                want = np.cumsum(rows, axis=0)[-1] / n  # sequential fp64 sum
                assert np.array_equal(mean, want), (b, hk, j)


# ------------------------------------------------------------ the decode

def _decode_case(orc, w, lengths=None, chunks=(1.0,), seed=0):
    inp = synth.make_decode_inputs(w, seed=seed, lengths=lengths)
    q, k, v, lengths = inp["q"], inp["k"], inp["v"], inp["lengths"]
    dt = synth.dtype_code(w.dtype)
    g_kv = _gkv(orc, k, v, lengths, dt)
    cache = _fill(k, v, lengths, w.capacity, g_kv, w.dtype, chunks=chunks, ss=w.use_scalesearch)
    need = ops.attn_decode_workspace_size(w.B, w.H, w.Hkv, w.capacity)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out, lse = ops.thrift_attn_decode(q.cuda(), cache, topk_frac=w.topk_frac,
                                      sink_blocks=w.sink_blocks, recent_blocks=w.recent_blocks,
                                      use_scalesearch=w.use_scalesearch, workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    r = orc.thrift_decode(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), dt,
                          np.array(lengths, np.int32), 128, g_kv, w.topk_frac,
                          use_ss=w.use_scalesearch, sink_blocks=w.sink_blocks,
                          recent_blocks=w.recent_blocks)
    nbcap = (w.capacity + 127) // 128
    mo = ops.attn_decode_mask_offset(w.B, w.H, w.Hkv, w.capacity)
    mask = ws[mo:mo + w.B * w.H * nbcap].cpu().numpy().reshape(w.B, w.H, nbcap)
    assert np.array_equal(mask, r["mask"]), np.argwhere(mask != r["mask"])[:5]
    _compare(out.float().cpu().numpy(), r["out64"], r["tol"], w.dtype)
    lg, lw = lse.cpu().numpy(), r["lse"]
    assert np.array_equal(np.isneginf(lg), np.isneginf(lw))
    fin = np.isfinite(lw)
    assert np.max(np.abs(lg[fin] - lw[fin]), initial=0.0) < 1e-2
    return mask


def _w(B, H, Hkv, capacity, frac, dtype=torch.bfloat16, ss=False, sink=0, recent=0):
    return synth.DecodeWorkload("case", B, H, Hkv, capacity, 1, capacity, 128, dtype, frac, ss,
                                sink_blocks=sink, recent_blocks=recent)


@pytest.mark.parametrize("H,Hkv", [(8, 2), (16, 2), (16, 1), (4, 4)], ids=["G4", "G8", "G16", "G1"])
def test_decode_mixed_selection(orc, H, Hkv):
    mask = _decode_case(orc, _w(3, H, Hkv, 1024, 0.3), lengths=[1000, 129, 1])
    assert mask.sum() > 0


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_decode_single_path(orc, frac):
    mask = _decode_case(orc, _w(2, 8, 2, 768, frac), lengths=[700, 256])
    nb = np.array([6, 2])
    assert mask.sum() == (0 if frac == 0.0 else 8 * nb.sum())


def test_decode_sink_recent_fp16_scalesearch(orc):
    _decode_case(orc, _w(2, 8, 2, 1024, 0.1, dtype=torch.float16, ss=True, sink=1, recent=1),
                 lengths=[1024, 385], chunks=(0.3, 0.6, 1.0))


def test_decode_empty_sequence(orc):
    _decode_case(orc, _w(3, 8, 2, 512, 0.25), lengths=[0, 300, 17])


def test_decode_many_splits(orc):
    # B * Hkv = 2: up to 32 CTAs per sequence, one or two tiles each
    _decode_case(orc, _w(1, 8, 2, 8192, 0.2), lengths=[8000])


def test_decode_few_splits(orc):
    # B * Hkv = 64: a few CTAs per sequence, many tiles each
    _decode_case(orc, _w(8, 16, 8, 2048, 0.1), lengths=None, seed=3)


def test_decode_full_size_sampled(orc):
    """The bench workload (Llama-3.1-8B attention shape, 131k context) in the
    launch the bench times; the oracle recomputes one sequence with the
    step's g_Q, kv scales and selection."""
    w = synth.C_DECODE131K
    inp = synth.make_decode_inputs(w, device="cuda")
    q, k, v, lengths = inp["q"], inp["k"], inp["v"], inp["lengths"]
    L = lengths[0]
    assert all(x == L for x in lengths)
    # the cache's scales g = amax / 2688 of the cached K and V (reading R1),
    # from the oracle on host copies, one batch entry at a time: the division
    # is correctly rounded and monotone, so the largest per-entry scale is the
    # scale of the whole tensor (no entry is all zero)
    g_kv = tuple(max(float(orc.tensor_scale(synth.as_u16(t[b, :L].cpu()).reshape(-1, 128), 1))
                     for b in range(w.B)) for t in (k, v))
    kv = torch.tensor(g_kv, dtype=torch.float32)
    cache = ops.DoubleKVCache(w.B, w.Hkv, w.capacity, kv, dtype=w.dtype)
    for t0 in range(0, L, 32768):
        t1 = min(L, t0 + 32768)
        cache.append(k[:, t0:t1].contiguous(), v[:, t0:t1].contiguous())
    need = ops.attn_decode_workspace_size(w.B, w.H, w.Hkv, w.capacity)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out, lse = ops.thrift_attn_decode(q, cache, topk_frac=w.topk_frac, workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    nbcap = (w.capacity + 127) // 128
    mo = ops.attn_decode_mask_offset(w.B, w.H, w.Hkv, w.capacity)
    mask = ws[mo:mo + w.B * w.H * nbcap].cpu().numpy().reshape(w.B, w.H, nbcap)
    qu = synth.as_u16(q.cpu())
    gq = float(orc.tensor_scale(qu.reshape(-1, 128), 1))
    b = 1
    r = orc.thrift_decode(qu[b:b + 1], synth.as_u16(k[b:b + 1].cpu()), synth.as_u16(v[b:b + 1].cpu()),
                          1, np.array([lengths[b]], np.int32), 128, g_kv, w.topk_frac, gq=gq)
    assert np.array_equal(mask[b:b + 1], r["mask"])
    _compare(out[b:b + 1].float().cpu().numpy(), r["out64"], r["tol"], w.dtype)
    assert np.max(np.abs(lse[b:b + 1].cpu().numpy() - r["lse"])) < 1e-2


def test_decode_long_context(orc):
    # 2049 key tiles: the selection's keys still fit the shared-memory cache,
    # the tile list spans several list-building rounds
    _decode_case(orc, _w(1, 4, 1, 2049 * 128, 0.05), lengths=[2049 * 128 - 77])


def test_decode_large_batch(orc):
    # a query tensor above the size reduced inside the query-image kernel:
    # the separate absmax kernel runs
    _decode_case(orc, _w(20, 16, 2, 512, 0.2), seed=5)
