"""CPU oracle for NVFP4 attention with selective FP16 block pairs.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It wraps the
plain C++ library ``liboracle.so`` built from ``oracle.cpp`` (see
``oracle/build.py``); it shares no code with the CUDA path.

Every function takes and returns numpy arrays.  16-bit tensors travel as
``uint16`` bit patterns plus a dtype code (0 = fp16, 1 = bf16).

The arithmetic, its sources and the readings taken where the pages are silent
are documented at the top of ``oracle.cpp``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from .build import build_oracle, LIB_PATH

_lib = None

F16, BF16 = 0, 1


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(
            os.path.join(os.path.dirname(LIB_PATH), "oracle.cpp")
        ):
            build_oracle()
        L = C.CDLL(LIB_PATH)
        P = C.c_void_p
        i64, i32, f32, u8 = C.c_int64, C.c_int, C.c_float, C.c_uint8
        L.orc_e2m1_encode.restype = u8
        L.orc_e2m1_encode.argtypes = [f32]
        L.orc_e2m1_decode.restype = f32
        L.orc_e2m1_decode.argtypes = [u8]
        L.orc_ue4m3_encode.restype = u8
        L.orc_ue4m3_encode.argtypes = [f32]
        L.orc_ue4m3_decode.restype = f32
        L.orc_ue4m3_decode.argtypes = [u8]
        L.orc_e2m1_encode_array.argtypes = [P, i64, P]
        L.orc_ue4m3_encode_array.argtypes = [P, i64, P]
        L.orc_half_to_float.restype = f32
        L.orc_half_to_float.argtypes = [C.c_uint16, i32]
        L.orc_double_to_half.restype = C.c_uint16
        L.orc_double_to_half.argtypes = [C.c_double, i32]
        L.orc_fwht_row.argtypes = [P, i32]
        L.orc_tensor_scale.restype = f32
        L.orc_tensor_scale.argtypes = [P, i32, i64, i64, i32]
        L.orc_block_err.restype = C.c_double
        L.orc_block_err.argtypes = [P, f32, u8]
        L.orc_quant_block.argtypes = [P, f32, i32, P, P, P]
        L.orc_nvfp4_quantize.restype = i32
        L.orc_nvfp4_quantize.argtypes = [P, i32, i64, i64, i32, i32, i32, P, P, P, P]
        L.orc_nvfp4_quantize_colblocks.restype = i32
        L.orc_nvfp4_quantize_colblocks.argtypes = [P, i32, i64, i64, i32, i32, P, P, P, P]
        L.orc_topk_count.restype = i64
        L.orc_topk_count.argtypes = [f32, i64]
        L.orc_block_mean_topk.restype = i32
        L.orc_block_mean_topk.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                          i32, P, P]
        L.orc_block_mean_topk_varlen.restype = i32
        L.orc_block_mean_topk_varlen.argtypes = [P, P, i32, i32, i32, P, i32, i32, i32, i32, f32,
                                                 i32, i32, P]
        L.orc_thrift_attn.restype = i32
        L.orc_thrift_attn.argtypes = [P, P, P, i32, i32, i32, P, i32, i32, i32, i32, f32, i32, i32,
                                      i32, i32, P, i32, P, i64, i32, P, P, P, P, P]
        L.orc_attn_fp64.restype = i32
        L.orc_attn_fp64.argtypes = [P, P, P, i32, i32, i32, P, i32, i32, i32, P, i64, i32, P, P]
        L.orc_thrift_attn_ex.restype = i32
        L.orc_thrift_attn_ex.argtypes = [P, P, P, i32, i32, i32, P, i32, i32, i32, i32, f32, i32,
                                         i32, i32, i32, i32, P, i32, P, i64, i32, P, P, P, P, P]
        L.orc_k_channel_means.argtypes = [P, i32, i32, P, i32, i32, P]
        L.orc_attn_qat_bwd.restype = i32
        L.orc_attn_qat_bwd.argtypes = [P, P, P, P, i32, i32, i32, P, i32, i32, i32, i32, i32, i32,
                                       P, P, P, P, P, P, P]
        L.orc_thrift_decode.restype = i32
        L.orc_thrift_decode.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, f32,
                                        i32, i32, i32, P, i32, P, i32, P, P, P, P, P]
        L.orc_thrift_attn_g.restype = i32
        L.orc_thrift_attn_g.argtypes = [P, P, P, i32, i32, i32, P, i32, i32, i32, i32, f32, i32,
                                        i32, i32, i32, i32, P, P, i32, P, i64, i32, P, P, P, P, P]
        L.orc_tensor_absmax.restype = f32
        L.orc_tensor_absmax.argtypes = [P, i32, i64, i64, i32]
        L.orc_set_test_hooks.restype = None
        L.orc_set_test_hooks.argtypes = [C.c_double, C.c_uint64, i32, i32, i32, i32, f32, i32]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _u16(x):
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, x.dtype
    return x


def nthreads_default():
    return max(1, os.cpu_count() or 1)


# ------------------------------------------------------------------ formats

def e2m1_encode(t):
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.empty(t.shape, np.uint8)
    lib().orc_e2m1_encode_array(_p(t), t.size, _p(out))
    return out


def e2m1_decode(codes):
    L = lib()
    return np.array([L.orc_e2m1_decode(int(c)) for c in np.ravel(codes)], np.float32).reshape(
        np.shape(codes))


def ue4m3_encode(v):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_ue4m3_encode_array(_p(v), v.size, _p(out))
    return out


def ue4m3_decode(b):
    L = lib()
    return np.array([L.orc_ue4m3_decode(int(c)) for c in np.ravel(b)], np.float32).reshape(
        np.shape(b))


def half_to_float(h, dt):
    L = lib()
    return np.array([L.orc_half_to_float(int(c), dt) for c in np.ravel(h)], np.float32).reshape(
        np.shape(h))


def double_to_half(x, dt):
    L = lib()
    return np.array([L.orc_double_to_half(float(c), dt) for c in np.ravel(x)], np.uint16).reshape(
        np.shape(x))


def fwht_rows(x):
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    for r in range(flat.shape[0]):
        lib().orc_fwht_row(_p(flat[r]), d)
    return x


# ---------------------------------------------------------------- quantiser

def block_err(x16, g, S):
    x16 = np.ascontiguousarray(x16, dtype=np.float32)
    assert x16.size == 16
    return lib().orc_block_err(_p(x16), float(g), int(S))


def quant_block(x16, g, use_ss):
    x16 = np.ascontiguousarray(x16, dtype=np.float32)
    codes = np.zeros(8, np.uint8)
    sc = np.zeros(1, np.uint8)
    f = np.zeros(1, np.int32)
    lib().orc_quant_block(_p(x16), float(g), int(use_ss), _p(codes), _p(sc), _p(f))
    return codes, int(sc[0]), int(f[0])


def tensor_scale(x, dt, hadamard=False):
    x = _u16(x)
    cols = x.shape[-1]
    return lib().orc_tensor_scale(_p(x), dt, x.size // cols, cols, int(hadamard))


def tensor_absmax(x, dt, hadamard=False):
    """max |x| over a [..., cols] 16-bit tensor (rows rotated first with
    hadamard)."""
    x = _u16(x)
    cols = x.shape[-1]
    return lib().orc_tensor_absmax(_p(x), dt, x.size // cols, cols, int(hadamard))


def scale_from_absmax(amax):
    """g = amax / 2688 in fp32 (1 for amax = 0), reading R1."""
    a = np.float32(amax)
    return float(np.float32(1.0)) if a == 0 else float(a / np.float32(2688.0))


def nvfp4_quantize(x, dt, use_ss=False, use_had=False, g=None):
    """Quantise a [rows, cols] 16-bit matrix, 16-blocks along cols.

    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16],
    g float, f int8 [rows, cols/16])."""
    x = _u16(x)
    cols = x.shape[-1]
    rows = x.size // cols
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    f = np.zeros((rows, cols // 16), np.int8)
    gg = np.array([g if g is not None else 0.0], np.float32)
    rc = lib().orc_nvfp4_quantize(_p(x), dt, rows, cols, int(use_ss), int(use_had),
                                  int(g is not None), _p(codes), _p(scales), _p(gg), _p(f))
    if rc:
        raise ValueError("oracle nvfp4_quantize: bad arguments")
    return codes, scales, float(gg[0]), f


def nvfp4_quantize_colblocks(x, dt, use_ss=False, g=None):
    """Quantise a [rows, cols] 16-bit matrix, 16-blocks along rows.

    Returns (codes [cols, rows/2], scales [cols, rows/16], g, f [cols, rows/16])."""
    x = _u16(x)
    rows, cols = x.shape
    codes = np.zeros((cols, rows // 2), np.uint8)
    scales = np.zeros((cols, rows // 16), np.uint8)
    f = np.zeros((cols, rows // 16), np.int8)
    gg = np.array([g if g is not None else 0.0], np.float32)
    rc = lib().orc_nvfp4_quantize_colblocks(_p(x), dt, rows, cols, int(use_ss), int(g is not None),
                                            _p(codes), _p(scales), _p(gg), _p(f))
    if rc:
        raise ValueError("oracle nvfp4_quantize_colblocks: bad arguments")
    return codes, scales, float(gg[0]), f


def dequantize(codes, scales, g):
    """Dequantised fp64 values of row-blocked codes [rows, cols/2]."""
    lo = codes & 0xF
    hi = codes >> 4
    c = np.stack([lo, hi], -1).reshape(codes.shape[0], -1)
    mags = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    vals = mags[c & 7] * np.where(c & 8, -1.0, 1.0)
    s = ue4m3_decode(scales).astype(np.float64)
    return vals * np.repeat(s, 16, axis=1) * float(g)


# ---------------------------------------------------------------- selection

def topk_count(frac, n_valid):
    return lib().orc_topk_count(float(frac), int(n_valid))


def block_mean_topk(q, k, dt, blk, causal, frac, sink_blocks=0, recent_blocks=0):
    """q [B,N,H,d], k [B,N,Hkv,d] uint16.  Returns (mask uint8 [B,H,nB,nB],
    scores fp64 [B,H,nB,nB]).  sink_blocks / recent_blocks: fixed FP16 pairs
    OR-ed with the top-k ones (reading R14 of oracle.cpp)."""
    q, k = _u16(q), _u16(k)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    nb = (N + blk - 1) // blk
    mask = np.zeros((B, H, nb, nb), np.uint8)
    scores = np.zeros((B, H, nb, nb), np.float64)
    rc = lib().orc_block_mean_topk(_p(q), _p(k), dt, B, H, Hkv, N, d, blk, int(causal),
                                   float(frac), int(sink_blocks), int(recent_blocks), _p(mask),
                                   _p(scores))
    if rc:
        raise ValueError("oracle block_mean_topk: bad arguments")
    return mask, scores


def block_mean_topk_varlen(q, k, dt, cu, blk, causal, frac, sink_blocks=0, recent_blocks=0):
    """q [total,H,d], k [total,Hkv,d]; cu int32 [nseq+1].  Returns the flat
    mask (per sequence [H, nB_s, nB_s], concatenated)."""
    q, k = _u16(q), _u16(k)
    cu = np.ascontiguousarray(cu, np.int32)
    H, d = q.shape[1], q.shape[2]
    Hkv = k.shape[1]
    lens = np.diff(cu)
    nbs = (lens + blk - 1) // blk
    mask = np.zeros(int(H * np.sum(nbs.astype(np.int64) ** 2)), np.uint8)
    rc = lib().orc_block_mean_topk_varlen(_p(q), _p(k), dt, H, Hkv, _p(cu), len(lens), d, blk,
                                          int(causal), float(frac), int(sink_blocks),
                                          int(recent_blocks), _p(mask))
    if rc:
        raise ValueError("oracle block_mean_topk_varlen: bad arguments")
    return mask


# ---------------------------------------------------------------- attention

def k_channel_means(k, dt, cu):
    """K channel means of reading R16: k [total, Hkv, d] -> fp32 [nseq, Hkv, d]."""
    k = _u16(k)
    cu = np.ascontiguousarray(cu, np.int32)
    total, Hkv, d = k.shape
    mu = np.zeros((len(cu) - 1, Hkv, d), np.float32)
    lib().orc_k_channel_means(_p(k), dt, Hkv, _p(cu), len(cu) - 1, d, _p(mu))
    return mu


def thrift_attn(q, k, v, dt, cu, blk, causal, frac, use_ss=False, use_had=False,
                mask=None, units=None, nthreads=None, sink_blocks=0, recent_blocks=0,
                smooth_k=False, g=None):
    """Emulated NVFP4 + FP16 attention over packed sequences.

    q [total,H,d], k/v [total,Hkv,d] uint16; cu int32 [nseq+1].
    Returns dict(out uint16 [total,H,d], out64 fp64 [total,H,d] (before the
    final rounding to the 16-bit type), tol fp64 [total,H,d] (bound on the
    effect of roundings that are not unique, see oracle.cpp), lse f32
    [H,total], mask flat uint8, g (g_Q, g_K, g_V)).  ``units``: optional int array [n,3] of
    (sequence, head, query block) to compute; other rows stay 0 / NaN.  ``g``: optional
    given (g_Q, g_K, g_V) (a shard of a larger problem), else computed (reading R1)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    cu = np.ascontiguousarray(cu, np.int32)
    total, H, d = q.shape
    Hkv = k.shape[1]
    lens = np.diff(cu)
    nbs = (lens + blk - 1) // blk
    msize = int(H * np.sum(nbs.astype(np.int64) ** 2))
    if mask is None:
        m = np.zeros(msize, np.uint8)
        given = 0
    else:
        m = np.ascontiguousarray(mask, np.uint8).reshape(-1).copy()
        assert m.size == msize
        given = 1
    out = np.zeros((total, H, d), np.uint16)
    out64 = np.zeros((total, H, d), np.float64)
    tol = np.zeros((total, H, d), np.float64)
    lse = np.full((H, total), np.nan, np.float32)
    gs = np.zeros(3, np.float32)
    if units is not None:
        u = np.ascontiguousarray(units, np.int32).reshape(-1, 3)
        n_units = u.shape[0]
    else:
        u, n_units = None, 0
    g_in = None if g is None else np.ascontiguousarray(g, np.float32).reshape(3)
    rc = lib().orc_thrift_attn_g(_p(q), _p(k), _p(v), dt, H, Hkv, _p(cu), len(lens), d, blk,
                                 int(causal), float(frac), int(sink_blocks), int(recent_blocks),
                                 int(use_ss), int(use_had), int(smooth_k), _p(g_in), _p(m), given,
                                 _p(u), n_units, int(nthreads or nthreads_default()), _p(out),
                                 _p(lse), _p(gs), _p(out64), _p(tol))
    if rc:
        raise ValueError("oracle thrift_attn: bad arguments")
    return {"out": out, "out64": out64, "tol": tol, "lse": lse, "mask": m,
            "g": tuple(float(x) for x in gs)}


def attn_fp64(q, k, v, dt, cu, causal, rows=None, nthreads=None):
    """Unquantised fp64 attention.  Returns (out fp64 [total,H,d], lse fp64
    [H,total]).  ``rows``: optional int64 [n,2] of (token, head)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    cu = np.ascontiguousarray(cu, np.int32)
    total, H, d = q.shape
    Hkv = k.shape[1]
    out = np.full((total, H, d), np.nan, np.float64)
    lse = np.full((H, total), np.nan, np.float64)
    if rows is not None:
        r = np.ascontiguousarray(rows, np.int64).reshape(-1, 2)
        n = r.shape[0]
    else:
        r, n = None, 0
    rc = lib().orc_attn_fp64(_p(q), _p(k), _p(v), dt, H, Hkv, _p(cu), len(cu) - 1, d,
                             int(causal), _p(r), n, int(nthreads or nthreads_default()), _p(out),
                             _p(lse))
    if rc:
        raise ValueError("oracle attn_fp64: bad arguments")
    return out, lse


# ------------------------------------------------------------------ decode

def thrift_decode(q, k, v, dt, lens, blk, g_kv, frac, use_ss=False, sink_blocks=0,
                  recent_blocks=0, mask=None, gq=None, nthreads=None):
    """One decode step over the double cache (reading R15 of oracle.cpp).

    q [B,H,d] uint16; k/v [B,ncap,Hkv,d] uint16 (token t of sequence b at
    [b, t]); lens int32 [B]; g_kv (g_K, g_V) floats.  Returns dict(out
    uint16 [B,H,d], out64 fp64 [B,H,d], tol fp64 [B,H,d], lse f32 [B,H],
    mask uint8 [B,H,nbcap], gq).  ``gq``: optional given g_Q (for a sample
    of the sequences of a larger step)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, H, d = q.shape
    ncap, Hkv = k.shape[1], k.shape[2]
    lens = np.ascontiguousarray(lens, np.int32)
    nbcap = (ncap + blk - 1) // blk
    if mask is None:
        m = np.zeros((B, H, nbcap), np.uint8)
        given = 0
    else:
        m = np.ascontiguousarray(mask, np.uint8).reshape(B, H, nbcap).copy()
        given = 1
    gkv = np.ascontiguousarray(g_kv, np.float32).reshape(2)
    out = np.zeros((B, H, d), np.uint16)
    out64 = np.zeros((B, H, d), np.float64)
    tol = np.zeros((B, H, d), np.float64)
    lse = np.full((B, H), np.nan, np.float32)
    gq_in = None if gq is None else np.array([gq], np.float32)
    gq_out = np.zeros(1, np.float32)
    rc = lib().orc_thrift_decode(_p(q), _p(k), _p(v), dt, B, H, Hkv, ncap, d, blk, _p(lens),
                                 _p(gkv), float(frac), int(sink_blocks), int(recent_blocks),
                                 int(use_ss), _p(m), given, _p(gq_in),
                                 int(nthreads or nthreads_default()), _p(out), _p(lse),
                                 _p(gq_out), _p(out64), _p(tol))
    if rc:
        raise ValueError("oracle thrift_decode: bad arguments")
    return {"out": out, "out64": out64, "tol": tol, "lse": lse, "mask": m,
            "gq": float(gq_out[0])}


# ---------------------------------------------------------- Attn-QAT bwd

def attn_qat_bwd(q, k, v, dout, dt, cu, blk, causal, use_ss=False, nthreads=None, g=None):
    """Attn-QAT forward outputs and gradients (reading R17 of oracle.cpp).

    q, dout [total,H,d], k, v [total,Hkv,d] uint16; cu int32 [nseq+1].
    g: optional tensor scales (gq, gk, gv) to use instead of those of the
    given tensors (a slice of a larger problem keeps the whole tensors').
    Returns dict(o, o_hp [total,H,d], lse [H,total], dq [total,H,d],
    dk, dv [total,Hkv,d]), all fp64."""
    q, k, v, dout = _u16(q), _u16(k), _u16(v), _u16(dout)
    cu = np.ascontiguousarray(cu, np.int32)
    total, H, d = q.shape
    Hkv = k.shape[1]
    o = np.zeros((total, H, d))
    o_hp = np.zeros((total, H, d))
    lse = np.zeros((H, total))
    dq = np.zeros((total, H, d))
    dk = np.zeros((total, Hkv, d))
    dv = np.zeros((total, Hkv, d))
    garr = None if g is None else np.ascontiguousarray(g, np.float32)
    rc = lib().orc_attn_qat_bwd(_p(q), _p(k), _p(v), _p(dout), dt, H, Hkv, _p(cu), len(cu) - 1, d,
                                blk, int(causal), int(use_ss), int(nthreads or nthreads_default()),
                                _p(garr) if garr is not None else None,
                                _p(o), _p(o_hp), _p(lse), _p(dq), _p(dk), _p(dv))
    if rc:
        raise ValueError("oracle attn_qat_bwd: bad arguments")
    return {"o": o, "o_hp": o_hp, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


# ------------------------------------------------------------ test hooks

class test_hooks:
    """Context manager that sets the emulation's test hooks (pins of the
    non-unique-rounding bound ``tol`` only; see oracle.cpp) and clears them
    on exit.  pert: every rounding input of the probabilities is multiplied by
    1 + pert * rho * u, u in [-1, 1) from a hash of (seed, position); plant:
    (sequence, head, row, key) whose scaled NVFP4 probability becomes plant_t
    and whose E2M1 code then moves ``force`` grid steps."""

    def __init__(self, pert=0.0, seed=0, plant=None, plant_t=0.0, force=0):
        self.args = (float(pert), int(seed)) + (tuple(plant) if plant else (-1, -1, -1, -1)) + (
            float(plant_t), int(force))

    def __enter__(self):
        lib().orc_set_test_hooks(*self.args)
        return self

    def __exit__(self, *exc):
        lib().orc_set_test_hooks(0.0, 0, -1, -1, -1, -1, 0.0, 0)
        return False

