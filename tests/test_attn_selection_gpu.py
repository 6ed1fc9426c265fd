"""The block-pair selection an attention call computes for itself
(ThriftAttention, Metodologia step 1: block means of Q and K, pair scores,
top-k per head) against the oracle's, bit for bit.  The attention path takes
the block means from its image kernels, so this is checked on its own and
not only through the standalone selection call.  The selection is read from
the caller-owned workspace at the offset the library reports."""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _mask_from_ws(ws, nseq, maxlen, H, Hkv, d, blk):
    off = ops.thrift_attn_workspace_mask_offset(nseq, maxlen, H, Hkv, d, blk)
    assert off > 0
    nB = (maxlen + blk - 1) // blk
    n = nseq * H * nB * nB
    return ws[off:off + n].cpu().numpy().reshape(nseq, H, nB, nB)


@pytest.mark.parametrize("name", ["tiny", "b2h32n8192", "gqa32k"])
def test_fixed_length(orc, name):
    w = {"tiny": synth.TINY, "b2h32n8192": synth.C_B2H32N8K, "gqa32k": synth.C_GQA32K}[name]
    inp = synth.make_attn_inputs(w)
    q, k, v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
    need = ops.thrift_attn_workspace_size(w.B, w.H, w.Hkv, w.N, w.d, w.blk)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=w.topk_frac,
                        use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                        workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    got = _mask_from_ws(ws, w.B, w.N, w.H, w.Hkv, w.d, w.blk)
    want, _ = orc.block_mean_topk(synth.as_u16(inp["q"]), synth.as_u16(inp["k"]),
                                  synth.dtype_code(w.dtype), w.blk, w.causal, w.topk_frac)
    assert np.array_equal(got, want), f"{np.argwhere(got != want)[:5]}"
    assert got.sum() > 0


@pytest.mark.parametrize("frac", [0.05, 0.25])
def test_varlen(orc, frac):
    import dataclasses
    w = dataclasses.replace(synth.C_VARLEN, topk_frac=frac)
    inp = synth.make_attn_inputs(w)
    q, k, v, cu = inp["q"], inp["k"], inp["v"], inp["cu_seqlens"]
    lengths = inp["lengths"]
    nseq, maxlen = len(lengths), max(lengths)
    need = ops.thrift_attn_varlen_workspace_size(nseq, q.shape[0], maxlen, w.H, w.Hkv, w.d, w.blk)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ops.thrift_attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), maxlen, blk=w.blk,
                               causal=w.causal, topk_frac=w.topk_frac,
                               use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                               workspace=ws)
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    got = _mask_from_ws(ws, nseq, maxlen, w.H, w.Hkv, w.d, w.blk)
    flat = orc.block_mean_topk_varlen(synth.as_u16(q), synth.as_u16(k), synth.dtype_code(w.dtype),
                                      cu.numpy(), w.blk, w.causal, w.topk_frac)
    pos = 0
    for s, L in enumerate(lengths):
        nb = (L + w.blk - 1) // w.blk
        want = flat[pos:pos + w.H * nb * nb].reshape(w.H, nb, nb)
        pos += w.H * nb * nb
        assert np.array_equal(got[s, :, :nb, :nb], want), f"sequence {s}"
