"""The C-ABI library loads on a machine without a GPU, exports every entry
point the header declares, and rejects bad arguments on the host before any
launch."""
import ctypes as C
import os
import re

import pytest

from bit_quantization_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*([a-z_][a-z0-9_]*)\s*\(",
                             text, flags=re.M):
            names.append(m.group(1))
    return names


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def test_every_declared_symbol_is_exported(L):
    names = _header_functions()
    assert len(names) >= 11
    assert set(names) == set(ops.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    assert ops.status_string(0) == "ok"
    assert ops.status_string(-4) == "device wait timed out"


def test_workspace_sizes_are_host_only(L):
    assert L.nvfp4_quantize_workspace_size() >= 16
    assert L.thrift_attn_workspace_size(1, 1, 1, 256, 64, 64) > 0
    assert L.thrift_attn_workspace_size(1, 1, 1, 256, 96, 64) == 0
    assert L.block_mean_topk_workspace_size(2, 32, 32, 8192, 128, 128) > 2 * 32 * 64 * 64 * 8
    big = L.thrift_attn_workspace_size(1, 32, 8, 32768, 128, 128)
    assert big < 1 << 31


def test_bad_arguments_rejected_before_launch(L):
    P = C.c_void_p
    dummy = P(4096)
    ws = P(8192)
    qws = L.nvfp4_quantize_workspace_size()
    # cols not a multiple of 16
    assert L.nvfp4_quantize(dummy, 0, 4, 24, 0, 0, 0, dummy, dummy, dummy, ws, qws, None) == ops.ERR_ARG
    # Hadamard on an unsupported width
    assert L.nvfp4_quantize(dummy, 0, 4, 32, 0, 1, 0, dummy, dummy, dummy, ws, qws, None) == ops.ERR_UNSUPPORTED
    # workspace too small
    assert L.nvfp4_quantize(dummy, 0, 4, 32, 0, 0, 0, dummy, dummy, dummy, ws, qws - 1, None) == ops.ERR_ARG
    # misaligned input
    assert L.nvfp4_quantize(P(4098), 0, 4, 32, 0, 0, 0, dummy, dummy, dummy, ws, qws, None) == ops.ERR_ARG
    # attention: unsupported head dim, bad GQA ratio, bad fraction, null pointer
    assert L.thrift_attn_fwd(dummy, dummy, dummy, 1, 1, 4, 4, 256, 96, 128, 0, C.c_float(0.1), 0, 0, 0, 0, 0,
                             dummy, dummy, ws, 1 << 40, None) == ops.ERR_UNSUPPORTED
    assert L.thrift_attn_fwd(dummy, dummy, dummy, 1, 1, 4, 3, 256, 128, 128, 0, C.c_float(0.1), 0, 0, 0, 0, 0,
                             dummy, dummy, ws, 1 << 40, None) == ops.ERR_ARG
    assert L.thrift_attn_fwd(dummy, dummy, dummy, 1, 1, 4, 4, 256, 128, 128, 0, C.c_float(1.5), 0, 0, 0, 0, 0,
                             dummy, dummy, ws, 1 << 40, None) == ops.ERR_ARG
    assert L.thrift_attn_fwd(None, dummy, dummy, 1, 1, 4, 4, 256, 128, 128, 0, C.c_float(0.1), 0, 0, 0, 0, 0,
                             dummy, dummy, ws, 1 << 40, None) == ops.ERR_ARG
    assert L.thrift_attn_fwd(dummy, dummy, dummy, 1, 1, 4, 4, 256, 128, 128, 0, C.c_float(0.1), 0, 0, 0, 0, 0,
                             dummy, dummy, ws, 16, None) == ops.ERR_ARG
    assert L.block_mean_topk(dummy, dummy, 0, 1, 4, 4, 256, 128, 32, 0, C.c_float(0.1), 0, 0, dummy, ws,
                             1 << 40, None) == ops.ERR_UNSUPPORTED
    assert L.thrift_attn_fwd_varlen(dummy, dummy, dummy, 1, None, 2, 100, 64, 4, 4, 128, 128, 1,
                                    C.c_float(0.1), 0, 0, 0, 0, 0, dummy, dummy, ws, 1 << 40,
                                    None) == ops.ERR_ARG
    # negative sink / recent block counts
    assert L.thrift_attn_fwd(dummy, dummy, dummy, 1, 1, 4, 4, 256, 128, 128, 0, C.c_float(0.1), -1, 0,
                             0, 0, 0, dummy, dummy, ws, 1 << 40, None) == ops.ERR_ARG
    # K smoothing with the Hadamard rotation: not supported
    assert L.thrift_attn_fwd(dummy, dummy, dummy, 1, 1, 4, 4, 256, 128, 128, 0, C.c_float(0.1), 0, 0,
                             0, 1, 1, dummy, dummy, ws, 1 << 40, None) == ops.ERR_UNSUPPORTED
    assert L.block_mean_topk(dummy, dummy, 0, 1, 4, 4, 256, 128, 128, 0, C.c_float(0.1), 0, -2, dummy,
                             ws, 1 << 40, None) == ops.ERR_ARG
    # decode: unsupported head dim / tile, too many heads per kv head, bad
    # fraction, cache too small, workspace too small
    big = 1 << 40
    assert L.thrift_kv_cache_size(2, 4, 1024, 64, 128) == 0
    assert L.thrift_kv_cache_size(2, 4, 1024, 128, 64) == 0
    csz = L.thrift_kv_cache_size(2, 4, 1000, 128, 128)
    assert csz == 2 * 4 * 8 * (9216 * 2 + 32768 * 2 + 1024)
    assert L.thrift_attn_decode_workspace_size(2, 68, 4, 1024, 128, 128) == 0
    assert L.thrift_attn_decode(dummy, 1, 2, 8, 4, 64, 128, 1024, dummy, big, dummy, dummy,
                                C.c_float(0.1), 0, 0, 0, dummy, dummy, ws, big, None) == ops.ERR_UNSUPPORTED
    assert L.thrift_attn_decode(dummy, 1, 2, 68, 4, 128, 128, 1024, dummy, big, dummy, dummy,
                                C.c_float(0.1), 0, 0, 0, dummy, dummy, ws, big, None) == ops.ERR_UNSUPPORTED
    assert L.thrift_attn_decode(dummy, 1, 2, 8, 3, 128, 128, 1024, dummy, big, dummy, dummy,
                                C.c_float(0.1), 0, 0, 0, dummy, dummy, ws, big, None) == ops.ERR_ARG
    assert L.thrift_attn_decode(dummy, 1, 2, 8, 4, 128, 128, 1024, dummy, big, dummy, dummy,
                                C.c_float(1.5), 0, 0, 0, dummy, dummy, ws, big, None) == ops.ERR_ARG
    assert L.thrift_attn_decode(dummy, 1, 2, 8, 4, 128, 128, 1024, dummy, 4096, dummy, dummy,
                                C.c_float(0.1), 0, 0, 0, dummy, dummy, ws, big, None) == ops.ERR_ARG
    assert L.thrift_attn_decode(dummy, 1, 2, 8, 4, 128, 128, 1024, dummy, big, dummy, dummy,
                                C.c_float(0.1), 0, 0, 0, dummy, dummy, ws, 4096, None) == ops.ERR_ARG
    assert L.thrift_attn_decode(dummy, 1, 2, 8, 4, 128, 128, 1024, dummy, big, dummy, dummy,
                                C.c_float(0.1), -1, 0, 0, dummy, dummy, ws, big, None) == ops.ERR_ARG
    assert L.thrift_kv_cache_append(dummy, dummy, 1, 2, 4, 128, 128, 1024, dummy, dummy, 4,
                                    dummy, 0, dummy, 16, None) == ops.ERR_ARG
    assert L.thrift_kv_cache_append(dummy, dummy, 1, 2, 4, 128, 128, 1024, dummy, dummy, -1,
                                    dummy, 0, dummy, big, None) == ops.ERR_ARG
    # nothing to append: accepted without a launch
    assert L.thrift_kv_cache_append(None, None, 1, 2, 4, 128, 128, 1024, dummy, dummy, 0,
                                    dummy, 0, dummy, big, None) == ops.OK
    # failure-detection aid: unknown mode, limits outside 1 us .. 1 s
    assert L.thrift_test_wait_timeout(2, 1000, None) == ops.ERR_ARG
    assert L.thrift_test_wait_timeout(0, 0, None) == ops.ERR_ARG
    assert L.thrift_test_wait_timeout(1, 1000001, None) == ops.ERR_ARG


def test_binding_fails_loudly_without_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    x = torch.zeros((16, 32), dtype=torch.float16)
    with pytest.raises(ops.ThriftError):
        ops.nvfp4_quantize(x)


def test_qat_entry_points_check_arguments_before_launch(L):
    """Attn-QAT: workspace size on the host, argument errors returned before
    any launch (no device needed)."""
    P = C.c_void_p
    dummy, ws, big = P(4096), P(8192), 1 << 40
    size = L.thrift_qat_workspace_size(1000, 2, 8, 2, 128)
    # 128-row tiles of Q, K, V and dO (1000 // 128 + 2 slots a head), 2 x
    # 16-byte scalars, D in fp32 (1024-byte slices)
    assert size >= (1000 // 128 + 2) * (8 + 2 + 2 + 8) * 128 * 128 * 2 + 1000 * 8 * 4
    assert L.thrift_qat_workspace_size(1000, 3, 8, 2, 128) > size
    assert L.thrift_qat_workspace_size(1000, 2, 8, 2, 96) == 0
    assert L.thrift_qat_workspace_size(0, 2, 8, 2, 128) == 0
    assert L.thrift_qat_workspace_size(1000, 0, 8, 2, 128) == 0

    def fwd(d=128, blk=128, H=8, Hkv=2, q=dummy, cu=dummy, wsb=big, out=dummy):
        return L.thrift_qat_fwd_varlen(q, dummy, dummy, 1, cu, 2, 1000, 600, H, Hkv, d, blk, 1, 0,
                                       out, dummy, dummy, ws, wsb, None)

    assert fwd(d=96) == ops.ERR_UNSUPPORTED
    assert fwd(blk=32) == ops.ERR_UNSUPPORTED
    assert fwd(Hkv=3) == ops.ERR_ARG
    assert fwd(q=None) == ops.ERR_ARG
    assert fwd(cu=None) == ops.ERR_ARG
    assert fwd(out=None) == ops.ERR_ARG
    assert fwd(q=P(4098)) == ops.ERR_ARG
    assert fwd(wsb=16) == ops.ERR_ARG

    def bwd(dout=dummy, dq=dummy, wsb=big):
        return L.thrift_qat_bwd_varlen(dummy, dummy, dummy, dout, 1, dummy, 2, 1000, 600, 8, 2, 128,
                                       128, 1, 0, 1, dummy, dummy, dq, dummy, dummy, ws, wsb, None)

    assert bwd(dout=None) == ops.ERR_ARG
    assert bwd(dq=None) == ops.ERR_ARG
    assert bwd(dq=P(4100)) == ops.ERR_ARG
    assert bwd(wsb=16) == ops.ERR_ARG


def test_binding_checks_shapes_before_the_device():
    """Mismatched inputs are rejected on the host with their shapes, before
    anything reaches a device (here: CPU tensors, so a consistent call only
    fails for want of a device)."""
    import torch
    bf = torch.bfloat16
    q = torch.zeros((1, 64, 4, 128), dtype=bf)
    k = torch.zeros((1, 64, 2, 128), dtype=bf)
    with pytest.raises(ops.ThriftError, match="differ"):
        ops.thrift_attn_fwd(q, k, torch.zeros((1, 64, 2, 64), dtype=bf))
    with pytest.raises(ops.ThriftError, match="differ outside the head axis"):
        ops.thrift_attn_fwd(q, torch.zeros((1, 32, 2, 128), dtype=bf), torch.zeros((1, 32, 2, 128), dtype=bf))
    with pytest.raises(ops.ThriftError, match="multiple of the kv heads"):
        ops.thrift_attn_fwd(q, torch.zeros((1, 64, 3, 128), dtype=bf), torch.zeros((1, 64, 3, 128), dtype=bf))
    with pytest.raises(ops.ThriftError, match="dtype"):
        ops.thrift_attn_fwd(q, k.half(), k.half())
    with pytest.raises(ops.ThriftError, match="lse must be"):
        ops.thrift_attn_fwd(q, k, k, lse=torch.zeros((1, 4, 32)))
    with pytest.raises(ops.ThriftError, match="dimensions"):
        ops.block_mean_topk(q[0], k[0], 64, False, 0.1)
    with pytest.raises(ops.ThriftError, match="cu_seqlens"):
        ops.thrift_attn_fwd_varlen(q[0], k[0], k[0], torch.zeros(3, dtype=torch.int64), 64)
    with pytest.raises(ops.ThriftError, match="dout must be"):
        ops.thrift_qat_bwd(q, k, k, q.half(), torch.zeros(q.shape), torch.zeros((4, 64)))
    with pytest.raises(ops.ThriftError, match="lse must be"):
        ops.thrift_qat_bwd(q, k, k, q, torch.zeros(q.shape), torch.zeros((4, 32)))
    # consistent shapes: only the device is missing
    if not torch.cuda.is_available():
        with pytest.raises(ops.ThriftError, match="CUDA device"):
            ops.thrift_attn_fwd(q, k, k)
        with pytest.raises(ops.ThriftError, match="CUDA device"):
            ops.thrift_qat_bwd(q, k, k, q, torch.zeros(q.shape), torch.zeros((4, 64)))


def test_quantiser_binding_checks_buffers_before_the_device():
    import torch
    x = torch.zeros((32, 64), dtype=torch.float16)
    with pytest.raises(ops.ThriftError, match=r"x must be \[rows, cols\]"):
        ops.nvfp4_quantize(x.reshape(2, 16, 64))
    with pytest.raises(ops.ThriftError, match="codes must be"):
        ops.nvfp4_quantize(x, codes=torch.zeros((32, 16), dtype=torch.uint8))
    with pytest.raises(ops.ThriftError, match="scales must be"):
        ops.nvfp4_quantize(x, scales=torch.zeros((32, 4), dtype=torch.int8))
    with pytest.raises(ops.ThriftError, match="tensor_scale"):
        ops.nvfp4_quantize_colblocks(x, tensor_scale=torch.zeros(1, dtype=torch.float16))
