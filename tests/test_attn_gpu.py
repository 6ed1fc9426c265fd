"""GPU attention vs the oracle's emulation of the same quantisation and
tiling (ThriftAttention Metodologia step 2; ScaleSearchAttention).

Bar (tests/parity_bars.py): |out - oracle| <= 1e-2 + half an ulp of the
16-bit output type + the oracle's bound for roundings that are not unique,
element by element, and cosine >= 0.9999, against the oracle's output before
its own final rounding; at most 0.1% of the elements may need that bound,
each in a row with a real midpoint.  lse within 1e-2.  Error against
unquantised fp64 attention is reported.
"""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops, synth
from parity_bars import MAX_ABS, MIN_COS, compare, half_ulp  # noqa: F401

pytestmark = pytest.mark.gpu


def _to_f(orc, u16, dt):
    return orc.half_to_float(u16, dt).astype(np.float64) if u16.size < 200000 else \
        _fast_f(u16, dt)


def _fast_f(u16, dt):
    t = torch.from_numpy(u16.view(np.int16))
    return (t.view(torch.bfloat16) if dt == 1 else t.view(torch.float16)).double().numpy()


def _compare(got, want64, what, dtype, tol=None):
    err, cos, _ = compare(got, want64, dtype, tol, what)
    return err, cos


def run_case(orc, B, N, H, Hkv, d, blk, causal, frac, ss, had, dtype, seed=0, k_off=3.0,
             sink=0, recent=0, smooth=False):
    w = synth.AttnWorkload("case", B, H, Hkv, N, d, dtype, causal, blk, frac, ss, had,
                           k_offset_std=k_off, seed=seed)
    inp = synth.make_attn_inputs(w)
    q, k, v = inp["q"], inp["k"], inp["v"]
    out, lse = ops.thrift_attn_fwd(q.cuda(), k.cuda(), v.cuda(), blk=blk, causal=causal,
                                   topk_frac=frac, use_scalesearch=ss, use_hadamard=had,
                                   sink_blocks=sink, recent_blocks=recent, smooth_k=smooth)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    dt = synth.dtype_code(dtype)
    cu = np.arange(B + 1, dtype=np.int32) * N
    qp, kp, vp = (synth.as_u16(t.reshape(B * N, -1, d)) for t in (q, k, v))
    r = orc.thrift_attn(qp, kp, vp, dt, cu, blk, causal, frac, use_ss=ss, use_had=had,
                        sink_blocks=sink, recent_blocks=recent, smooth_k=smooth)
    got = out.cpu().reshape(B * N, H, d)
    gotf = got.double().numpy()
    _compare(gotf, r["out64"], "out", dtype, r["tol"])
    lse_want = r["lse"].reshape(H, B, N).transpose(1, 0, 2)
    assert np.max(np.abs(lse.cpu().numpy() - lse_want)) < 1e-2
    return gotf, qp, kp, vp, cu, dt


def test_tiny_workload(orc):
    w = synth.TINY
    gotf, qp, kp, vp, cu, dt = run_case(orc, w.B, w.N, w.H, w.Hkv, w.d, w.blk, w.causal,
                                        w.topk_frac, w.use_scalesearch, w.use_hadamard, w.dtype,
                                        k_off=0.0)
    ref, _ = orc.attn_fp64(qp, kp, vp, dt, cu, w.causal)
    print("tiny: max abs error vs fp64 attention", np.max(np.abs(gotf - ref)))


CASES = [
    # B, N, H, Hkv, d, blk, causal, frac, ss, had, dtype
    (1, 384, 2, 1, 128, 128, False, 0.0, False, False, torch.bfloat16),
    (2, 300, 4, 2, 128, 128, True, 0.25, True, True, torch.bfloat16),
    (1, 200, 2, 2, 64, 64, True, 0.5, False, True, torch.float16),
    (1, 256, 2, 2, 64, 128, False, 1.0, False, False, torch.float16),
    (1, 520, 2, 1, 128, 64, True, 0.1, True, False, torch.bfloat16),
    (1, 129, 1, 1, 128, 128, True, 0.05, False, False, torch.float16),
    (3, 17, 2, 2, 64, 64, False, 0.3, True, True, torch.bfloat16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c[:10]))
def test_parity_cases(orc, case):
    run_case(orc, *case)


def test_varlen_parity(orc):
    lens = [100, 257, 384, 1, 129]
    H, Hkv, d, blk = 4, 2, 128, 128
    total = sum(lens)
    gen = torch.Generator().manual_seed(7)
    q = torch.randn((total, H, d), generator=gen).to(torch.bfloat16)
    k = (torch.randn((total, Hkv, d), generator=gen) + 2.0).to(torch.bfloat16)
    v = torch.randn((total, Hkv, d), generator=gen).to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cu_t = torch.from_numpy(cu).cuda()
    for frac, ss, had, smooth in [(0.0, False, False, False), (0.25, True, True, False),
                                  (1.0, False, True, False), (0.25, False, False, True)]:
        out, lse = ops.thrift_attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_t, max(lens),
                                              blk=blk, causal=True, topk_frac=frac,
                                              use_scalesearch=ss, use_hadamard=had,
                                              smooth_k=smooth)
        torch.cuda.synchronize()
        assert ops.device_status(reset=True) == ops.OK
        r = orc.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), 1, cu, blk, True,
                            frac, use_ss=ss, use_had=had, smooth_k=smooth)
        _compare(out.cpu().double().numpy(), r["out64"], f"varlen frac={frac}", torch.bfloat16,
                 r["tol"])
        assert np.max(np.abs(lse.cpu().numpy() - r["lse"])) < 1e-2


SINK_CASES = [
    # B, N, H, Hkv, d, blk, causal, frac, ss, had, dtype, sink, recent
    (1, 640, 2, 1, 128, 128, True, 0.1, True, True, torch.bfloat16, 1, 1),
    (1, 512, 2, 2, 128, 128, False, 0.0, False, False, torch.bfloat16, 1, 1),
    (2, 300, 2, 1, 64, 64, True, 0.05, False, True, torch.float16, 2, 2),
]


@pytest.mark.parametrize("case", SINK_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_sink_blocks_parity(orc, case):
    # ScaleSearchAttention's sink-aware mixed precision: the first and the
    # most recent key blocks on the FP16 path, on top of the top-k pairs
    *args, sink, recent = case
    run_case(orc, *args, sink=sink, recent=recent)


def test_all_fp16_pairs_match_fp64(orc):
    # topk_frac = 1: every pair on the FP16 path -> plain 16-bit attention.
    gotf, qp, kp, vp, cu, dt = run_case(orc, 1, 256, 2, 2, 128, 128, True, 1.0, False, False,
                                        torch.float16)
    ref, _ = orc.attn_fp64(qp, kp, vp, dt, cu, True)
    assert np.max(np.abs(gotf.reshape(ref.shape) - ref)) < 4e-3


def test_deterministic():
    inp = synth.make_attn_inputs(synth.TINY)
    a = ops.thrift_attn_fwd(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), blk=64,
                            topk_frac=0.25)[0]
    b = ops.thrift_attn_fwd(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), blk=64,
                            topk_frac=0.25)[0]
    assert torch.equal(a, b)


SMOOTH_CASES = [
    # B, N, H, Hkv, d, blk, causal, frac, ss, dtype, K channel-offset std
    (1, 384, 2, 1, 128, 128, False, 0.0, False, torch.bfloat16, 20.0),
    (2, 300, 4, 2, 128, 128, True, 0.25, True, torch.bfloat16, 20.0),
    (1, 520, 2, 1, 128, 64, True, 0.1, False, torch.float16, 8.0),
    (1, 200, 2, 2, 64, 64, False, 0.5, True, torch.bfloat16, 3.0),
]


@pytest.mark.parametrize("case", SMOOTH_CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_k_smoothing_parity(orc, case):
    B, N, H, Hkv, d, blk, causal, frac, ss, dtype, k_off = case
    run_case(orc, B, N, H, Hkv, d, blk, causal, frac, ss, False, dtype, k_off=k_off, smooth=True)


def test_k_smoothing_improves_accuracy():
    """Under strong K channel offsets the NVFP4 path loses most of K's
    resolution to the offset; smoothing takes it back (error against fp64
    attention at least halved)."""
    import oracle as orc_mod
    w = synth.AttnWorkload("case", 1, 4, 2, 1024, 128, torch.bfloat16, True, 128, 0.1, False,
                           False, k_offset_std=20.0, seed=3)
    inp = synth.make_attn_inputs(w)
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    errs = []
    cu = np.array([0, w.N], np.int32)
    ref, _ = orc_mod.attn_fp64(synth.as_u16(inp["q"][0]), synth.as_u16(inp["k"][0]),
                               synth.as_u16(inp["v"][0]), 1, cu, True)
    for smooth in (False, True):
        out, _ = ops.thrift_attn_fwd(q, k, v, blk=128, causal=True, topk_frac=0.1,
                                     smooth_k=smooth)
        torch.cuda.synchronize()
        errs.append(float(np.sqrt(np.mean((out[0].double().cpu().numpy() - ref) ** 2))))
    assert ops.device_status(reset=True) == ops.OK
    assert errs[1] < 0.5 * errs[0], errs
