"""One attention problem split by (batch entry, kv-head group) on the GPU
(ThriftAttention Metodologia step 1: all but the per-tensor scales is per
(sequence, head)).  The ranks are emulated one after another on one device:
each shard's thrift_attn_absmax, their elementwise maximum (what the ranks'
max all-reduce computes), then each shard's thrift_attn_fwd_absmax.  Every
shard's output, LSE and selection must equal the matching slice of the
one-call run bit for bit, and the agreed absmaxes those of the whole
problem."""
import pytest
import torch

from bit_quantization_b200 import ops, shard, synth

pytestmark = pytest.mark.gpu

CASES = [
    # B, N, H, Hkv, d, blk, causal, frac, ss, had, world
    (2, 1000, 8, 4, 128, 128, True, 0.05, True, True, 2),
    (2, 1000, 8, 4, 128, 128, True, 0.05, True, True, 4),
    (4, 384, 4, 4, 64, 64, False, 0.25, False, False, 8),
    (2, 520, 8, 2, 128, 128, True, 0.1, False, False, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(str(x) for x in c))
def test_shards_match_the_whole_problem(case):
    B, N, H, Hkv, d, blk, causal, frac, ss, had, world = case
    w = synth.AttnWorkload("shard", B, H, Hkv, N, d, torch.bfloat16, causal, blk, frac, ss, had,
                           k_offset_std=3.0, seed=9)
    inp = synth.make_attn_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    ws = torch.empty(ops.thrift_attn_workspace_size(B, H, Hkv, N, d, blk), dtype=torch.uint8,
                     device="cuda")
    out, lse = ops.thrift_attn_fwd(q, k, v, blk=blk, causal=causal, topk_frac=frac,
                                   use_scalesearch=ss, use_hadamard=had, workspace=ws)
    nB = (N + blk - 1) // blk
    mo = ops.thrift_attn_workspace_mask_offset(B, N, H, Hkv, d, blk)
    mask = ws[mo:mo + B * H * nB * nB].view(B, H, nB, nB).clone()
    whole = ops.thrift_attn_absmax(q, k, v, blk=blk, use_hadamard=had).clone()
    shards = [shard.shard_of(B, H, Hkv, world, r) for r in range(world)]
    parts = [tuple(shard.take(t, s, kv=i > 0) for i, t in enumerate((q, k, v))) for s in shards]
    amaxes = [ops.thrift_attn_absmax(*p, blk=blk, use_hadamard=had).clone() for p in parts]
    agreed = torch.stack(amaxes).amax(dim=0)
    assert torch.equal(agreed, whole)
    for s, p in zip(shards, parts):
        Bs, Hs, Hkvs = s.b1 - s.b0, s.h1 - s.h0, s.hk1 - s.hk0
        wss = torch.empty(ops.thrift_attn_varlen_workspace_size(Bs, Bs * N, N, Hs, Hkvs, d, blk),
                          dtype=torch.uint8, device="cuda")
        o_s, l_s = ops.thrift_attn_fwd_absmax(*p, agreed, blk=blk, causal=causal, topk_frac=frac,
                                              use_scalesearch=ss, use_hadamard=had,
                                              workspace=wss)
        torch.cuda.synchronize()
        assert ops.stream_status(reset=True) == ops.OK
        assert torch.equal(o_s, out[s.b0:s.b1, :, s.h0:s.h1])
        assert torch.equal(l_s, lse[s.b0:s.b1, s.h0:s.h1])
        mo_s = ops.thrift_attn_workspace_mask_offset(Bs, N, Hs, Hkvs, d, blk)
        m_s = wss[mo_s:mo_s + Bs * Hs * nB * nB].view(Bs, Hs, nB, nB)
        assert torch.equal(m_s, mask[s.b0:s.b1, s.h0:s.h1])


def test_varlen_heads_split():
    lens = [300, 1, 900, 129]
    H, Hkv, d, blk = 8, 4, 128, 128
    total = sum(lens)
    gen = torch.Generator().manual_seed(13)
    q = torch.randn((total, H, d), generator=gen).to(torch.bfloat16).cuda()
    k = (torch.randn((total, Hkv, d), generator=gen) + 1.5).to(torch.bfloat16).cuda()
    v = torch.randn((total, Hkv, d), generator=gen).to(torch.bfloat16).cuda()
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32).cuda()
    mx = max(lens)
    out, lse = ops.thrift_attn_fwd_varlen(q, k, v, cu, mx, blk=blk, causal=True, topk_frac=0.2,
                                          use_scalesearch=True, use_hadamard=True)
    parts = [(q[:, :4].contiguous(), k[:, :2].contiguous(), v[:, :2].contiguous()),
             (q[:, 4:].contiguous(), k[:, 2:].contiguous(), v[:, 2:].contiguous())]
    amax = torch.stack([ops.thrift_attn_absmax(*p, cu, mx, blk=blk, use_hadamard=True).clone()
                        for p in parts]).amax(dim=0)
    for i, p in enumerate(parts):
        o_s, l_s = ops.thrift_attn_fwd_absmax(*p, amax, cu, mx, blk=blk, causal=True,
                                              topk_frac=0.2, use_scalesearch=True,
                                              use_hadamard=True)
        torch.cuda.synchronize()
        assert torch.equal(o_s, out[:, 4 * i:4 * i + 4])
        assert torch.equal(l_s, lse[4 * i:4 * i + 4])
    assert ops.stream_status(reset=True) == ops.OK
