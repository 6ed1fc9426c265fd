"""GPU block selection vs the oracle (ThriftAttention, Metodologia step 1):
the selected block-pair sets must be bit-identical."""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _check(orc, q, k, blk, causal, frac):
    mask = ops.block_mean_topk(q.cuda(), k.cuda(), blk, causal, frac).cpu().numpy()
    m0, _ = orc.block_mean_topk(synth.as_u16(q), synth.as_u16(k), synth.dtype_code(q.dtype), blk,
                                causal, frac)
    assert np.array_equal(mask, m0), f"{np.argwhere(mask != m0)[:5]}"
    return mask


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("frac", [0.0, 0.1, 0.3, 1.0])
def test_small_parity(orc, causal, frac):
    q = synth.randn16((2, 1000, 4, 128), torch.bfloat16, 1)
    k = (synth.randn16((2, 1000, 2, 128), torch.float32, 2) + 1.5).to(torch.bfloat16)
    _check(orc, q, k, 128, causal, frac)


def test_tiny_workload(orc):
    inp = synth.make_attn_inputs(synth.TINY)
    m = _check(orc, inp["q"], inp["k"], 64, False, 0.25)
    assert m.sum() == 4


def test_ties_lower_index():
    q = torch.ones((1, 256, 1, 64), dtype=torch.float16, device="cuda")
    k = torch.ones((1, 256, 1, 64), dtype=torch.float16, device="cuda")
    m = ops.block_mean_topk(q, k, 64, False, 0.25).cpu().numpy().reshape(-1)
    assert m[:4].all() and not m[4:].any()


@pytest.mark.parametrize("w", [synth.C_B2H32N8K, synth.C_GQA32K], ids=lambda w: w.name)
def test_full_size_workloads(orc, w):
    inp = synth.make_attn_inputs(w)
    m = _check(orc, inp["q"], inp["k"], w.blk, w.causal, w.topk_frac)
    nb = w.N // w.blk
    n_valid = nb * (nb + 1) // 2 if w.causal else nb * nb
    assert (m.reshape(w.B * w.H, -1).sum(1) == orc.topk_count(w.topk_frac, n_valid)).all()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("frac,sink,recent", [(0.0, 1, 1), (0.1, 1, 2), (0.3, 3, 0), (1.0, 1, 1)])
def test_sink_blocks_parity(orc, causal, frac, sink, recent):
    # ScaleSearchAttention's sink-aware pairs OR-ed with the top-k selection
    q = synth.randn16((2, 1000, 4, 128), torch.bfloat16, 5)
    k = (synth.randn16((2, 1000, 2, 128), torch.float32, 6) + 1.5).to(torch.bfloat16)
    mask = ops.block_mean_topk(q.cuda(), k.cuda(), 128, causal, frac, sink_blocks=sink,
                               recent_blocks=recent).cpu().numpy()
    m0, _ = orc.block_mean_topk(synth.as_u16(q), synth.as_u16(k), synth.dtype_code(q.dtype), 128,
                                causal, frac, sink_blocks=sink, recent_blocks=recent)
    assert np.array_equal(mask, m0), f"{np.argwhere(mask != m0)[:5]}"
