"""The no-allocation selection entry point against the regular one.

block_mean_topk_noalloc serves callers that cannot allocate device memory
(code running under CUDA graph capture, or a plug-in that only receives
tensors and a stream from a framework owning all device memory); its scratch
is a fixed array inside the library.  Its selection must equal the regular
entry point's bit for bit (the selection tests' bar), on two calls in a row,
the second with different inputs so stale scratch contents would show.
This file is collected last so a failure here leaves every other test run.
"""
import pytest
import torch

from bit_quantization_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _inputs(seed, B=2, N=1000, H=4, Hkv=2, d=128):
    q = synth.randn16((B, N, H, d), torch.bfloat16, seed).cuda()
    k = (synth.randn16((B, N, Hkv, d), torch.float32, seed + 1) + 1.5).to(torch.bfloat16).cuda()
    return q, k


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_regular_twice(causal):
    for call, (seed, frac) in enumerate([(31, 0.1), (47, 0.3)]):
        q, k = _inputs(seed)
        want = ops.block_mean_topk(q, k, 128, causal, frac)
        got = ops.block_mean_topk_noalloc(q, k, 128, causal, frac)
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"call {call}: selection differs"


def test_noalloc_tiny_workload():
    inp = synth.make_attn_inputs(synth.TINY)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    for _ in range(2):
        got = ops.block_mean_topk_noalloc(q, k, 64, False, 0.25)
        want = ops.block_mean_topk(q, k, 64, False, 0.25)
        assert torch.equal(got, want)


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, H, Hkv, N, d, blk = 1, 32, 8, 32768, 128, 128
    assert ops.lib().block_mean_topk_workspace_size(B, H, Hkv, N, d, blk) > ops.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, N, H, d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, N, Hkv, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.ThriftError, match="fixed scratch"):
        ops.block_mean_topk_noalloc(q, k, blk, True, 0.05)
