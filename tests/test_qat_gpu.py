"""Attn-QAT forward and backward ("Attn-QAT", Metodologia 1 and 2) through
the C ABI against the oracle's reading R17, element by element.

Tolerance, from the arithmetic: the GPU path computes in fp32 with P, its
FP4 image and dS rounded to the 16-bit input type before the tensor-core
products (relative 2^-9 for bf16, 2^-12 for fp16, with fp32 accumulation),
and takes the same FP4 code decisions from fp32 probabilities, so an
occasional code at a rounding boundary may differ from the fp64 oracle's.
Each tensor must agree within 1e-2 of its largest reference magnitude (for
the outputs O and O', within 1e-2 absolute when that magnitude is below 1)
and have cosine similarity >= 0.9999 with it -- the forward's parity bar
(max-abs 1e-2, cosine 0.9999) applied to each output and gradient on its
own scale.  lse agrees within 1e-3 absolute."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from bit_quantization_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _close(name, got, want, rel=1e-2, cos=0.9999):
    got = np.asarray(got, np.float64).ravel()
    want = np.asarray(want, np.float64).ravel()
    assert np.isfinite(got).all(), f"{name}: non-finite output"
    scale = max(float(np.abs(want).max()), 1.0e-30)
    err = float(np.abs(got - want).max())
    assert err <= rel * max(scale, 1.0 if name in ("o", "o_hp") else scale), \
        f"{name}: max abs err {err:.3e} vs scale {scale:.3e}"
    den = float(np.sqrt((got * got).sum() * (want * want).sum()))
    if den > 0:
        c = float((got * want).sum()) / den
        assert c >= cos, f"{name}: cosine {c:.6f}"


def _run_gpu(inp, w, reuse=False):
    q, k, v, dout = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    cu = inp["cu_seqlens"].cuda()
    maxlen = max(inp["lengths"])
    ws = torch.empty(ops.qat_workspace_size(q.shape[0], w.H, w.Hkv, w.d, cu.numel() - 1),
                     dtype=torch.uint8, device="cuda")
    out, out_hp, lse = ops.thrift_qat_fwd(q, k, v, cu, maxlen, blk=w.blk, causal=w.causal,
                                          use_scalesearch=w.use_scalesearch, workspace=ws)
    dq, dk, dv = ops.thrift_qat_bwd(q, k, v, dout, out_hp, lse, cu, maxlen, blk=w.blk,
                                    causal=w.causal, use_scalesearch=w.use_scalesearch,
                                    reuse_images=reuse, workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    return {"o": out.float().cpu().numpy(), "o_hp": out_hp.cpu().numpy(),
            "lse": lse.cpu().numpy(), "dq": dq.cpu().numpy(), "dk": dk.cpu().numpy(),
            "dv": dv.cpu().numpy()}


def _run_oracle(inp, w, g=None):
    u = {n: synth.as_u16(inp[n]) for n in ("q", "k", "v", "dout")}
    return oracle.attn_qat_bwd(u["q"], u["k"], u["v"], u["dout"], synth.dtype_code(w.dtype),
                               inp["cu_seqlens"].numpy(), w.blk, w.causal,
                               use_ss=w.use_scalesearch, g=g)


def _compare(got, want):
    for n in ("o", "o_hp", "dq", "dk", "dv"):
        _close(n, got[n], want[n])
    assert np.abs(got["lse"] - want["lse"]).max() <= 1e-3


CASES = {
    # name: (dtype, H, Hkv, d, blk, causal, scalesearch, lengths)
    "bf16_gqa_causal_varlen": (torch.bfloat16, 4, 2, 128, 128, True, False, [300, 130, 77]),
    "bf16_noncausal_blk64_ss": (torch.bfloat16, 2, 2, 128, 64, False, True, [200]),
    "fp16_d64_causal": (torch.float16, 2, 1, 64, 128, True, False, [257, 64]),
    "fp16_d64_blk64_noncausal": (torch.float16, 1, 1, 64, 64, False, False, [129]),
    "bf16_single_tokens": (torch.bfloat16, 2, 1, 128, 128, True, False, [1, 17, 1, 64]),
}


@pytest.mark.parametrize("name", list(CASES))
def test_qat_matches_oracle(name):
    dt, H, Hkv, d, blk, causal, ss, lengths = CASES[name]
    w = synth.QatWorkload(name, 1, H, Hkv, max(lengths), d, dt, causal, blk, ss, seed=11)
    inp = synth.make_qat_inputs(w, lengths=lengths)
    _compare(_run_gpu(inp, w), _run_oracle(inp, w))


@pytest.mark.parametrize("causal", [True, False])
def test_rising_scores_move_the_reference_maximum(causal):
    """Scores that grow by about 6 (natural units) per 128-key tile: every
    key tile's row maximum passes the previous one by more than 2^8, so the
    forward rescales O and O' at nearly every tile; results still match the
    oracle."""
    H, Hkv, d, N = 2, 1, 128, 640
    gen = torch.Generator().manual_seed(21)
    u = torch.randn(d, generator=gen)
    u = u / u.norm() * d ** 0.5
    a = (6.0 / d ** 0.5) ** 0.5
    t = torch.arange(N, dtype=torch.float32)[:, None, None] / 128.0
    q = a * u + 0.2 * torch.randn((N, H, d), generator=gen)
    k = a * t * u + 0.2 * torch.randn((N, Hkv, d), generator=gen)
    v = torch.randn((N, Hkv, d), generator=gen)
    dout = torch.randn((N, H, d), generator=gen)
    inp = {"q": q.to(torch.bfloat16), "k": k.to(torch.bfloat16), "v": v.to(torch.bfloat16),
           "dout": dout.to(torch.bfloat16), "cu_seqlens": torch.tensor([0, N], dtype=torch.int32),
           "lengths": [N]}
    w = synth.QatWorkload("rising", 1, H, Hkv, N, d, torch.bfloat16, causal, 128, False, seed=21)
    got, want = _run_gpu(inp, w), _run_oracle(inp, w)
    # the scores really do climb by more than 8 (log2) from tile to tile
    s = (q[:, 0].double() @ k[:, 0].double().T) / d ** 0.5
    tile_max = torch.stack([s[:, j:j + 128].max() for j in range(0, N, 128)])
    assert float((tile_max[1:] - tile_max[:-1]).min()) * 1.4427 > 8.0
    _compare(got, want)


def test_reused_images_give_the_same_gradients():
    dt, H, Hkv, d, blk, causal, ss, lengths = CASES["bf16_gqa_causal_varlen"]
    w = synth.QatWorkload("reuse", 1, H, Hkv, max(lengths), d, dt, causal, blk, True, seed=5)
    inp = synth.make_qat_inputs(w, lengths=lengths)
    a = _run_gpu(inp, w, reuse=False)
    b = _run_gpu(inp, w, reuse=True)
    for n in a:
        assert np.array_equal(a[n], b[n]), n
    _compare(b, _run_oracle(inp, w))


def test_fixed_length_batch_layout():
    """[B, N, H, d] inputs give the same results as their packed form."""
    w = synth.QatWorkload("fixed", 2, 2, 1, 192, 128, torch.bfloat16, True, 128, False, seed=2)
    inp = synth.make_qat_inputs(w, lengths=[192, 192])
    q, k, v, dout = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    out, out_hp, lse = ops.thrift_qat_fwd(q.view(2, 192, 2, 128), k.view(2, 192, 1, 128),
                                          v.view(2, 192, 1, 128), blk=128, causal=True)
    dq, dk, dv = ops.thrift_qat_bwd(q.view(2, 192, 2, 128), k.view(2, 192, 1, 128),
                                    v.view(2, 192, 1, 128), dout.view(2, 192, 2, 128), out_hp,
                                    lse, blk=128, causal=True)
    torch.cuda.synchronize()
    got = {"o": out.reshape(384, 2, 128).float().cpu().numpy(),
           "o_hp": out_hp.reshape(384, 2, 128).cpu().numpy(), "lse": lse.cpu().numpy(),
           "dq": dq.reshape(384, 2, 128).cpu().numpy(), "dk": dk.reshape(384, 1, 128).cpu().numpy(),
           "dv": dv.reshape(384, 1, 128).cpu().numpy()}
    _compare(got, _run_oracle(inp, w))


def test_full_size_sampled_kv_group():
    """The Attn-QAT bench workload (B1 H32 Hkv8 N4096 d128 bf16 causal) in
    the launch configuration the bench times; the oracle recomputes kv head 0
    with its four query heads, under the whole tensors' scales."""
    w = synth.C_QAT4K
    inp = synth.make_qat_inputs(w)
    got = _run_gpu(inp, w)
    dc = synth.dtype_code(w.dtype)
    g = tuple(oracle.tensor_scale(synth.as_u16(inp[n]), dc) for n in ("q", "k", "v"))
    grp = w.H // w.Hkv
    sl = {n: inp[n][:, :grp].contiguous() for n in ("q", "dout")}
    sl.update({n: inp[n][:, :1].contiguous() for n in ("k", "v")})
    sl["cu_seqlens"], sl["lengths"] = inp["cu_seqlens"], inp["lengths"]
    want = _run_oracle(sl, dataclasses.replace(w, H=grp, Hkv=1), g=g)
    part = {"o": got["o"][:, :grp], "o_hp": got["o_hp"][:, :grp], "lse": got["lse"][:grp],
            "dq": got["dq"][:, :grp], "dk": got["dk"][:, :1], "dv": got["dv"][:, :1]}
    _compare(part, want)


def test_rejects_bad_arguments():
    q = torch.zeros(64, 2, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(64, 1, 128, dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, 64], dtype=torch.int32, device="cuda")
    with pytest.raises(ops.ThriftError):
        ops.thrift_qat_fwd(q, k, k, cu, 64, blk=32)
    with pytest.raises(ops.ThriftError):
        ops.thrift_qat_fwd(q[:, :, :96].contiguous(), k[:, :, :96].contiguous(),
                           k[:, :, :96].contiguous(), cu, 64)
    with pytest.raises(ops.ThriftError):
        ops.thrift_qat_bwd(q, k, k, q, torch.zeros(64, 2, 128, device="cuda"),
                           torch.zeros(2, 64, device="cuda"), cu, 64, reuse_images=True)
