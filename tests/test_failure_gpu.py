"""Failure detection without a GPU fault: every device-side wait of the
library is bounded in wall time; one that gives up sets the device status
word (THRIFT_ERR_TIMEOUT), the kernel returns normally and the context stays
usable.  The waits are made to run out on purpose by the library's own aid,
which waits on an mbarrier that nothing arrives on, or on a global word that
nothing writes, with a limit of a few milliseconds."""
import time

import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [0, 1], ids=["mbarrier", "global_word"])
def test_bounded_wait_sets_timeout_status(mode):
    assert ops.device_status(reset=True) == ops.OK
    t0 = time.perf_counter()
    ops.test_wait_timeout(mode, 20000)  # 20 ms
    got = ops.device_status(reset=True)
    elapsed = time.perf_counter() - t0
    assert got == ops.ERR_TIMEOUT
    assert elapsed < 5.0
    # the word was cleared and the context still works
    assert ops.device_status() == ops.OK
    x = torch.randn(64, 64, device="cuda").to(torch.float16)
    codes, scales, g = ops.nvfp4_quantize(x)
    torch.cuda.synchronize()
    assert ops.device_status() == ops.OK
    assert codes.shape == (64, 32) and scales.shape == (64, 4)
    assert np.isfinite(float(g.item() if torch.is_tensor(g) else g))


def test_status_word_is_sticky_until_reset():
    assert ops.device_status(reset=True) == ops.OK
    ops.test_wait_timeout(0, 1000)
    assert ops.device_status() == ops.ERR_TIMEOUT  # read without reset
    assert ops.device_status(reset=True) == ops.ERR_TIMEOUT
    assert ops.device_status() == ops.OK


def test_attention_after_a_timeout():
    """A timed-out wait in one kernel does not disturb later calls."""
    ops.test_wait_timeout(1, 5000)
    assert ops.device_status(reset=True) == ops.ERR_TIMEOUT
    torch.manual_seed(0)
    q = torch.randn(1, 256, 2, 128, device="cuda").to(torch.bfloat16)
    k = torch.randn(1, 256, 2, 128, device="cuda").to(torch.bfloat16)
    v = torch.randn(1, 256, 2, 128, device="cuda").to(torch.bfloat16)
    out, lse = ops.thrift_attn_fwd(q, k, v, blk=128, topk_frac=0.25)
    torch.cuda.synchronize()
    assert ops.device_status() == ops.OK
    assert torch.isfinite(out.float()).all()


def test_stream_status_waits_for_its_own_stream_only():
    """thrift_stream_status synchronises one stream: while a bounded wait of
    300 ms runs on stream A, a status read through stream B returns at once
    (OK: the wait has not given up yet); the read through A waits for it and
    reports the timeout, and its reset clears the word."""
    assert ops.device_status(reset=True) == ops.OK
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(a):
        ops.test_wait_timeout(0, 300000)
    t0 = time.perf_counter()
    got_b = ops.stream_status(b)
    t_b = time.perf_counter() - t0
    got_a = ops.stream_status(a, reset=True)
    t_a = time.perf_counter() - t0
    assert got_b == ops.OK and t_b < 0.2, (got_b, t_b)
    assert got_a == ops.ERR_TIMEOUT and t_a >= 0.25, (got_a, t_a)
    assert ops.stream_status(b) == ops.OK
    assert ops.device_status() == ops.OK
