"""ctypes binding of libthrift_nvfp4.so (C ABI in include/thrift_nvfp4.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory and the current stream.  There is no
fallback: a missing library, a missing CUDA device or a failing call raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libthrift_nvfp4.so")

OK, ERR_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_SCRATCH = 0, -1, -2, -3, -4, -5
NOALLOC_SCRATCH_BYTES = 8 << 20
F16, BF16 = 0, 1

_lib = None

# Exported names of the C ABI, in header order.
EXPORTS = (
    "thrift_status_string", "thrift_device_status", "thrift_stream_status",
    "nvfp4_quantize_workspace_size",
    "nvfp4_quantize", "nvfp4_quantize_colblocks", "block_mean_topk_workspace_size",
    "block_mean_topk", "block_mean_topk_noalloc", "thrift_attn_workspace_size", "thrift_attn_fwd",
    "thrift_attn_varlen_workspace_size", "thrift_attn_fwd_varlen",
    "thrift_attn_absmax", "thrift_attn_fwd_absmax", "thrift_attn_workspace_mask_offset",
    "thrift_kernel_timer_enable", "thrift_kernel_timer_read", "thrift_test_wait_timeout",
    "thrift_kv_cache_size", "thrift_kv_cache_append", "thrift_attn_decode_workspace_size",
    "thrift_attn_decode_mask_offset", "thrift_attn_decode",
    "thrift_qat_workspace_size", "thrift_qat_fwd_varlen", "thrift_qat_bwd_varlen",
)


class ThriftError(RuntimeError):
    pass


def lib():
    """Loads the library (once).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ThriftError(
                "libthrift_nvfp4.so is not built; run `python -m bit_quantization_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, i32, i64, f32, sz = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t
        L.thrift_status_string.restype = C.c_char_p
        L.thrift_status_string.argtypes = [i32]
        L.thrift_device_status.restype = i32
        L.thrift_device_status.argtypes = [i32]
        L.thrift_stream_status.restype = i32
        L.thrift_stream_status.argtypes = [P, i32]
        L.nvfp4_quantize_workspace_size.restype = sz
        L.nvfp4_quantize_workspace_size.argtypes = []
        L.nvfp4_quantize.restype = i32
        L.nvfp4_quantize.argtypes = [P, i32, i64, i64, i32, i32, i32, P, P, P, P, sz, P]
        L.nvfp4_quantize_colblocks.restype = i32
        L.nvfp4_quantize_colblocks.argtypes = [P, i32, i64, i64, i32, i32, P, P, P, P, sz, P]
        L.block_mean_topk_workspace_size.restype = sz
        L.block_mean_topk_workspace_size.argtypes = [i32] * 6
        L.block_mean_topk.restype = i32
        L.block_mean_topk.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32, i32,
                                      P, P, sz, P]
        L.block_mean_topk_noalloc.restype = i32
        L.block_mean_topk_noalloc.argtypes = [P, P, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                              i32, i32, P, P]
        L.thrift_attn_workspace_size.restype = sz
        L.thrift_attn_workspace_size.argtypes = [i32] * 6
        L.thrift_attn_fwd.restype = i32
        L.thrift_attn_fwd.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                                      i32, i32, i32, i32, P, P, P, sz, P]
        L.thrift_attn_varlen_workspace_size.restype = sz
        L.thrift_attn_varlen_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32]
        L.thrift_attn_absmax.restype = i32
        L.thrift_attn_absmax.argtypes = [P, P, P, i32, P, i32, i64, i32, i32, i32, i32, i32, i32,
                                         i32, P, P, sz, P]
        L.thrift_attn_fwd_absmax.restype = i32
        L.thrift_attn_fwd_absmax.argtypes = [P, P, P, i32, P, i32, i64, i32, i32, i32, i32, i32,
                                             i32, f32, i32, i32, i32, i32, i32, P, P, P, P, sz, P]
        L.thrift_attn_workspace_mask_offset.restype = sz
        L.thrift_attn_workspace_mask_offset.argtypes = [i32, i32, i32, i32, i32, i32]
        L.thrift_attn_fwd_varlen.restype = i32
        L.thrift_attn_fwd_varlen.argtypes = [P, P, P, i32, P, i32, i64, i32, i32, i32, i32, i32,
                                             i32, f32, i32, i32, i32, i32, i32, P, P, P, sz, P]
        L.thrift_kernel_timer_enable.restype = i32
        L.thrift_kernel_timer_enable.argtypes = [i32]
        L.thrift_kernel_timer_read.restype = i32
        L.thrift_kernel_timer_read.argtypes = [P, P]
        L.thrift_test_wait_timeout.restype = i32
        L.thrift_test_wait_timeout.argtypes = [i32, i32, P]
        L.thrift_kv_cache_size.restype = sz
        L.thrift_kv_cache_size.argtypes = [i32] * 5
        L.thrift_kv_cache_append.restype = i32
        L.thrift_kv_cache_append.argtypes = [P, P, i32, i32, i32, i32, i32, i32, P, P, i32, P, i32,
                                             P, sz, P]
        L.thrift_attn_decode_workspace_size.restype = sz
        L.thrift_attn_decode_workspace_size.argtypes = [i32] * 6
        L.thrift_attn_decode_mask_offset.restype = sz
        L.thrift_attn_decode_mask_offset.argtypes = [i32] * 6
        L.thrift_attn_decode.restype = i32
        L.thrift_attn_decode.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, P, sz, P, P, f32,
                                         i32, i32, i32, P, P, P, sz, P]
        L.thrift_qat_workspace_size.restype = sz
        L.thrift_qat_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        L.thrift_qat_fwd_varlen.restype = i32
        L.thrift_qat_fwd_varlen.argtypes = [P, P, P, i32, P, i32, i64, i32, i32, i32, i32, i32,
                                            i32, i32, P, P, P, P, sz, P]
        L.thrift_qat_bwd_varlen.restype = i32
        L.thrift_qat_bwd_varlen.argtypes = [P, P, P, P, i32, P, i32, i64, i32, i32, i32, i32, i32,
                                            i32, i32, i32, P, P, P, P, P, P, sz, P]
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().thrift_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != OK:
        raise ThriftError(f"{what}: {status_string(code)} ({code})")


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise ThriftError(f"unsupported dtype {t.dtype}")


def _check_qkv(q, k, v=None, packed=False):
    """Shapes and dtypes of attention inputs, checked before anything reaches
    the device: q [B,N,H,d] (packed: [total,H,d]), k and v [B,N,Hkv,d]
    ([total,Hkv,d]) in one 16-bit type, H a multiple of Hkv."""
    nd = 3 if packed else 4
    ts = [("q", q), ("k", k)] + ([("v", v)] if v is not None else [])
    for name, t in ts:
        if t.dim() != nd:
            raise ThriftError(f"{name} must have {nd} dimensions, got {tuple(t.shape)}")
        if t.dtype != q.dtype:
            raise ThriftError(f"{name} has dtype {t.dtype}, q has {q.dtype}")
    _dt(q)
    if v is not None and v.shape != k.shape:
        raise ThriftError(f"v {tuple(v.shape)} and k {tuple(k.shape)} differ")
    if q.shape[:-2] != k.shape[:-2] or q.shape[-1] != k.shape[-1]:
        raise ThriftError(f"q {tuple(q.shape)} and k {tuple(k.shape)} differ outside the head axis")
    if k.shape[-2] <= 0 or q.shape[-2] % k.shape[-2]:
        raise ThriftError("the query heads must be a multiple of the kv heads")


def _check_like(t, shape, dtype, name):
    """A caller-supplied output or auxiliary tensor of a given shape and type."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ThriftError(f"{name} must be {dtype} of shape {tuple(shape)}, got {t.dtype} "
                          f"{tuple(t.shape)}")


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ThriftError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ThriftError("tensors must be contiguous")


def _stream(t: torch.Tensor):
    return C.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return C.c_void_p(t.data_ptr()) if t is not None else None


def device_status(reset: bool = False) -> int:
    """Synchronises the device; returns OK or ERR_TIMEOUT (device wait gave up)."""
    return lib().thrift_device_status(int(reset))


def stream_status(stream: Optional[torch.cuda.Stream] = None, reset: bool = False) -> int:
    """Waits for ``stream`` only (default: the current stream) and returns the
    device status word (OK or ERR_TIMEOUT), clearing it when ``reset``."""
    st = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.device(st.device):
        return lib().thrift_stream_status(C.c_void_p(st.cuda_stream), int(reset))


def _on(t: torch.Tensor):
    """Makes the tensor's device current around a library call (the library
    resolves per-device state, such as the no-allocation scratch address, on
    the current device)."""
    return torch.cuda.device(t.device)


def kernel_timer_enable(enable: bool):
    _check(lib().thrift_kernel_timer_enable(int(enable)), "thrift_kernel_timer_enable")


def kernel_timer_read():
    """Returns (summed attention-kernel milliseconds, timed launches)."""
    ms = C.c_double(0.0)
    n = C.c_int(0)
    _check(lib().thrift_kernel_timer_read(C.byref(ms), C.byref(n)), "thrift_kernel_timer_read")
    return ms.value, n.value


def test_wait_timeout(mode: int, limit_us: int, device=None):
    """Failure-detection aid: launches a kernel whose bounded wait (mode 0 an
    mbarrier nothing arrives on, mode 1 a global word nothing writes) gives
    up after ``limit_us`` and sets the device status word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    st = C.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    _check(lib().thrift_test_wait_timeout(int(mode), int(limit_us), st),
           "thrift_test_wait_timeout")


class Workspace:
    """Grow-only device scratch buffers reused across calls, one per (device,
    stream): a call uses the buffer of the stream it is queued on, so calls on
    different streams never share scratch, and a buffer that grows is freed
    back to the one stream that used it (allocated while that stream is
    current, so the caching allocator reuses it only in that stream's order)."""

    def __init__(self):
        self.bufs = {}

    def get(self, nbytes: int, device) -> torch.Tensor:
        nbytes = max(int(nbytes), 256)
        device = torch.device(device)
        stream = torch.cuda.current_stream(device)
        key = (device.index, stream.cuda_stream)
        buf = self.bufs.get(key)
        if buf is None or buf.numel() < nbytes:
            self.bufs.pop(key, None)
            with torch.cuda.device(device), torch.cuda.stream(stream):
                buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
            self.bufs[key] = buf
        return buf


_ws = Workspace()
_qws = Workspace()  # the quantiser's (needs no initial contents)


# ------------------------------------------------------------------ quantiser

def nvfp4_quantize(x: torch.Tensor, use_scalesearch=False, use_hadamard=False,
                   tensor_scale: Optional[torch.Tensor] = None, codes=None, scales=None,
                   workspace: Optional[torch.Tensor] = None):
    """x [rows, cols] fp16/bf16 on CUDA -> (codes u8 [rows, cols/2],
    scales u8 [rows, cols/16], tensor_scale f32 [1])."""
    if x.dim() != 2:
        raise ThriftError(f"x must be [rows, cols], got {tuple(x.shape)}")
    rows, cols = x.shape
    _check_like(codes, (rows, cols // 2), torch.uint8, "codes")
    _check_like(scales, (rows, cols // 16), torch.uint8, "scales")
    if tensor_scale is not None and (tensor_scale.dtype != torch.float32 or
                                     tensor_scale.numel() < 1):
        raise ThriftError("tensor_scale must be float32 with at least one element")
    _need_cuda(x)
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    given = tensor_scale is not None
    ts = tensor_scale if given else torch.empty(1, dtype=torch.float32, device=x.device)
    ws = workspace if workspace is not None else _qws.get(lib().nvfp4_quantize_workspace_size(),
                                                          x.device)
    with _on(x):
        _check(lib().nvfp4_quantize(_ptr(x), _dt(x), rows, cols, int(use_scalesearch),
                                    int(use_hadamard), int(given), _ptr(codes), _ptr(scales),
                                    _ptr(ts), _ptr(ws), ws.numel(), _stream(x)), "nvfp4_quantize")
    return codes, scales, ts


def nvfp4_quantize_colblocks(x: torch.Tensor, use_scalesearch=False,
                             tensor_scale: Optional[torch.Tensor] = None):
    """x [rows, cols] -> (codes [cols, rows/2], scales [cols, rows/16], g)."""
    if x.dim() != 2:
        raise ThriftError(f"x must be [rows, cols], got {tuple(x.shape)}")
    if tensor_scale is not None and (tensor_scale.dtype != torch.float32 or
                                     tensor_scale.numel() < 1):
        raise ThriftError("tensor_scale must be float32 with at least one element")
    _need_cuda(x)
    rows, cols = x.shape
    codes = torch.empty((cols, rows // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((cols, rows // 16), dtype=torch.uint8, device=x.device)
    given = tensor_scale is not None
    ts = tensor_scale if given else torch.empty(1, dtype=torch.float32, device=x.device)
    ws = _qws.get(lib().nvfp4_quantize_workspace_size(), x.device)
    with _on(x):
        _check(lib().nvfp4_quantize_colblocks(_ptr(x), _dt(x), rows, cols, int(use_scalesearch),
                                              int(given), _ptr(codes), _ptr(scales), _ptr(ts),
                                              _ptr(ws), ws.numel(), _stream(x)),
               "nvfp4_quantize_colblocks")
    return codes, scales, ts


# ------------------------------------------------------------------ selection

def block_mean_topk(q: torch.Tensor, k: torch.Tensor, blk: int, causal: bool, topk_frac: float,
                    sink_blocks: int = 0, recent_blocks: int = 0):
    """q [B,N,H,d], k [B,N,Hkv,d] -> mask u8 [B,H,nB,nB] (1 = FP16 pair).
    sink_blocks / recent_blocks: fixed FP16 key blocks added to the top-k
    pairs (see the header)."""
    _check_qkv(q, k)
    _need_cuda(q, k)
    B, N, H, d = q.shape
    Hkv = k.shape[2]
    nB = (N + blk - 1) // blk
    mask = torch.empty((B, H, nB, nB), dtype=torch.uint8, device=q.device)
    need = lib().block_mean_topk_workspace_size(B, H, Hkv, N, d, blk)
    ws = _ws.get(need, q.device)
    with _on(q):
        _check(lib().block_mean_topk(_ptr(q), _ptr(k), _dt(q), B, H, Hkv, N, d, blk, int(causal),
                                     float(topk_frac), int(sink_blocks), int(recent_blocks),
                                     _ptr(mask), _ptr(ws), ws.numel(), _stream(q)),
               "block_mean_topk")
    return mask


def block_mean_topk_noalloc(q: torch.Tensor, k: torch.Tensor, blk: int, causal: bool,
                            topk_frac: float, mask: Optional[torch.Tensor] = None,
                            sink_blocks: int = 0, recent_blocks: int = 0):
    """block_mean_topk with the library's fixed scratch instead of a workspace,
    for callers that cannot allocate device memory (see the header).  Pass
    `mask` to avoid the one allocation this wrapper would otherwise make."""
    _check_qkv(q, k)
    B, N, H, d = q.shape
    nB = (N + blk - 1) // blk
    _check_like(mask, (B, H, nB, nB), torch.uint8, "mask")
    _need_cuda(q, k)
    Hkv = k.shape[2]
    if mask is None:
        mask = torch.empty((B, H, nB, nB), dtype=torch.uint8, device=q.device)
    with _on(q):
        _check(lib().block_mean_topk_noalloc(_ptr(q), _ptr(k), _dt(q), B, H, Hkv, N, d, blk,
                                             int(causal), float(topk_frac), int(sink_blocks),
                                             int(recent_blocks), _ptr(mask), _stream(q)),
               "block_mean_topk_noalloc")
    return mask


# ------------------------------------------------------------------ attention

def thrift_attn_workspace_size(B, H, Hkv, N, d, blk) -> int:
    return int(lib().thrift_attn_workspace_size(B, H, Hkv, N, d, blk))


def thrift_attn_fwd(q, k, v, blk=128, causal=False, topk_frac=0.0, use_scalesearch=False,
                    use_hadamard=False, out=None, lse=None, workspace=None, sink_blocks=0,
                    recent_blocks=0, smooth_k=False):
    """q [B,N,H,d], k/v [B,N,Hkv,d] -> (out [B,N,H,d], lse f32 [B,H,N])."""
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    _check_like(out, q.shape, q.dtype, "out")
    _check_like(lse, (B, H, N), torch.float32, "lse")
    _need_cuda(q, k, v)
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    need = thrift_attn_workspace_size(B, H, Hkv, N, d, blk)
    if need == 0:
        raise ThriftError("thrift_attn_fwd: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, H, Hkv, N, d, blk,
                                     int(causal), float(topk_frac), int(sink_blocks),
                                     int(recent_blocks), int(use_scalesearch), int(use_hadamard),
                                     int(smooth_k), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                     _stream(q)),
               "thrift_attn_fwd")
    return out, lse


def thrift_attn_workspace_mask_offset(nseq, max_seqlen, H, Hkv, d, blk) -> int:
    """Byte offset of the selection mask [nseq, H, nB, nB] inside an attention
    workspace (valid once the call that used the workspace has completed)."""
    return int(lib().thrift_attn_workspace_mask_offset(nseq, max_seqlen, H, Hkv, d, blk))


def thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H, Hkv, d, blk) -> int:
    return int(lib().thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H, Hkv, d, blk))


def thrift_attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, blk=128, causal=True,
                           topk_frac=0.0, use_scalesearch=False, use_hadamard=False, out=None,
                           lse=None, workspace=None, sink_blocks=0, recent_blocks=0,
                           smooth_k=False):
    """q [total,H,d], k/v [total,Hkv,d], cu_seqlens int32 [nseq+1] (CUDA) ->
    (out [total,H,d], lse f32 [H,total])."""
    _check_qkv(q, k, v, packed=True)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ThriftError("cu_seqlens must be int32 [nseq + 1]")
    _check_like(out, q.shape, q.dtype, "out")
    _check_like(lse, (q.shape[1], q.shape[0]), torch.float32, "lse")
    _need_cuda(q, k, v, cu_seqlens)
    total, H, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    need = thrift_attn_varlen_workspace_size(nseq, total, max_seqlen, H, Hkv, d, blk)
    if need == 0:
        raise ThriftError("thrift_attn_fwd_varlen: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _dt(q), _ptr(cu_seqlens),
                                            nseq, total, int(max_seqlen), H, Hkv, d, blk,
                                            int(causal), float(topk_frac), int(sink_blocks),
                                            int(recent_blocks), int(use_scalesearch),
                                            int(use_hadamard), int(smooth_k), _ptr(out), _ptr(lse),
                                            _ptr(ws), ws.numel(), _stream(q)),
               "thrift_attn_fwd_varlen")
    return out, lse


def _shape_of(q, k, cu_seqlens, max_seqlen):
    """(nseq, total, max_seqlen, H, Hkv, d) of [B,N,H,d] or packed inputs."""
    if q.dim() == 4:
        B, N, H, d = q.shape
        return B, B * N, N, H, k.shape[2], d
    if cu_seqlens is None or max_seqlen is None:
        raise ThriftError("packed inputs need cu_seqlens and max_seqlen")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ThriftError("cu_seqlens must be int32 [nseq + 1]")
    total, H, d = q.shape
    return cu_seqlens.numel() - 1, total, int(max_seqlen), H, k.shape[1], d


def thrift_attn_absmax(q, k, v, cu_seqlens=None, max_seqlen=None, blk=128, use_hadamard=False,
                       smooth_k=False, amax=None, workspace=None):
    """The three tensor absmaxes (Q, K rotated when use_hadamard, V) of an
    attention call's inputs: float32 [3] on the device.  q [B,N,H,d] or
    packed [total,H,d] with cu_seqlens / max_seqlen."""
    _check_qkv(q, k, v, packed=q.dim() == 3)
    _need_cuda(q, k, v)
    nseq, total, maxlen, H, Hkv, d = _shape_of(q, k, cu_seqlens, max_seqlen)
    _check_like(amax, (3,), torch.float32, "amax")
    if amax is None:
        amax = torch.empty(3, dtype=torch.float32, device=q.device)
    need = thrift_attn_varlen_workspace_size(nseq, total, maxlen, H, Hkv, d, blk)
    if need == 0:
        raise ThriftError("thrift_attn_absmax: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_attn_absmax(_ptr(q), _ptr(k), _ptr(v), _dt(q), _ptr(cu_seqlens), nseq,
                                        total, maxlen, H, Hkv, d, blk, int(use_hadamard),
                                        int(smooth_k), _ptr(amax), _ptr(ws), ws.numel(),
                                        _stream(q)),
               "thrift_attn_absmax")
    return amax


def thrift_attn_fwd_absmax(q, k, v, amax, cu_seqlens=None, max_seqlen=None, blk=128,
                           causal=False, topk_frac=0.0, use_scalesearch=False, use_hadamard=False,
                           out=None, lse=None, workspace=None, sink_blocks=0, recent_blocks=0,
                           smooth_k=False):
    """thrift_attn_fwd (q [B,N,H,d]; lse [B,H,N]) or thrift_attn_fwd_varlen
    (packed, cu_seqlens; lse [H,total]) with the three tensor absmaxes given
    (float32 [3] on the device, e.g. agreed across the shards of a problem)."""
    _check_qkv(q, k, v, packed=q.dim() == 3)
    nseq, total, maxlen, H, Hkv, d = _shape_of(q, k, cu_seqlens, max_seqlen)
    lse_shape = (H, total) if q.dim() == 3 else (nseq, H, maxlen)
    _check_like(amax, (3,), torch.float32, "amax")
    _check_like(out, q.shape, q.dtype, "out")
    _check_like(lse, lse_shape, torch.float32, "lse")
    _need_cuda(q, k, v, amax)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    need = thrift_attn_varlen_workspace_size(nseq, total, maxlen, H, Hkv, d, blk)
    if need == 0:
        raise ThriftError("thrift_attn_fwd_absmax: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_attn_fwd_absmax(_ptr(q), _ptr(k), _ptr(v), _dt(q), _ptr(cu_seqlens),
                                            nseq, total, maxlen, H, Hkv, d, blk, int(causal),
                                            float(topk_frac), int(sink_blocks),
                                            int(recent_blocks), int(use_scalesearch),
                                            int(use_hadamard), int(smooth_k), _ptr(amax),
                                            _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                            _stream(q)),
               "thrift_attn_fwd_absmax")
    return out, lse


# ---------------------------------------------------------------- decode --

def kv_cache_size(B, Hkv, capacity, d=128, blk=128) -> int:
    return int(lib().thrift_kv_cache_size(B, Hkv, capacity, d, blk))


def attn_decode_workspace_size(B, H, Hkv, capacity, d=128, blk=128) -> int:
    return int(lib().thrift_attn_decode_workspace_size(B, H, Hkv, capacity, d, blk))


def attn_decode_mask_offset(B, H, Hkv, capacity, d=128, blk=128) -> int:
    return int(lib().thrift_attn_decode_mask_offset(B, H, Hkv, capacity, d, blk))


class DoubleKVCache:
    """The FP4 + 16-bit KV cache of ``B`` sequences (ThriftAttention decode):
    one zero-filled device buffer in the library's format, the cached lengths
    (int32, device) and the per-tensor scales (g_K, g_V) the NVFP4 part is
    quantised with."""

    def __init__(self, B, Hkv, capacity, kv_scale, dtype=torch.bfloat16, device="cuda",
                 d=128, blk=128, use_scalesearch=False):
        need = kv_cache_size(B, Hkv, capacity, d, blk)
        if need == 0:
            raise ThriftError("DoubleKVCache: unsupported shape")
        self.B, self.Hkv, self.capacity, self.d, self.blk = B, Hkv, capacity, d, blk
        self.dtype, self.use_scalesearch = dtype, use_scalesearch
        self.buf = torch.zeros(need, dtype=torch.uint8, device=device)
        self.lengths = torch.zeros(B, dtype=torch.int32, device=device)
        self.kv_scale = torch.as_tensor(kv_scale, dtype=torch.float32, device=device).reshape(2)

    def append(self, k_new, v_new, n_new=None, cache_len=None):
        """k_new, v_new [B, T, Hkv, d]; n_new int32 [B] (default: T each).
        ``cache_len`` (int32 [B], device): the positions to write at, for a
        caller that keeps its own lengths (``self.lengths`` is then left as
        it is); by default ``self.lengths``, advanced by ``n_new``."""
        if (k_new.dim() != 4 or k_new.shape != v_new.shape or k_new.shape[0] != self.B
                or k_new.shape[2] != self.Hkv or k_new.shape[3] != self.d):
            raise ThriftError(f"k_new, v_new must both be [B={self.B}, T, {self.Hkv}, {self.d}]")
        if k_new.dtype != self.dtype or v_new.dtype != self.dtype:
            raise ThriftError(f"k_new, v_new must be {self.dtype}")
        _need_cuda(k_new, v_new)
        B, T, Hkv, d = k_new.shape
        if n_new is None:
            n_new = torch.full((B,), T, dtype=torch.int32, device=k_new.device)
        at = self.lengths if cache_len is None else cache_len
        with _on(k_new):
            _check(lib().thrift_kv_cache_append(_ptr(k_new), _ptr(v_new), _dt(k_new), B, Hkv, d,
                                                self.blk, self.capacity, _ptr(at), _ptr(n_new), T,
                                                _ptr(self.kv_scale), int(self.use_scalesearch),
                                                _ptr(self.buf), self.buf.numel(), _stream(k_new)),
                   "thrift_kv_cache_append")
        if cache_len is None:
            self.lengths.add_(n_new)
            self.lengths.clamp_(max=self.capacity)


def thrift_attn_decode(q, cache: DoubleKVCache, topk_frac=0.0, sink_blocks=0, recent_blocks=0,
                       use_scalesearch=False, out=None, lse=None, workspace=None, seq_len=None):
    """q [B,H,d] -> (out [B,H,d], lse f32 [B,H]) against ``cache``
    (``seq_len``: int32 [B] device lengths to attend over instead of
    ``cache.lengths``)."""
    if q.dim() != 3 or q.shape[0] != cache.B or q.shape[2] != cache.d or q.shape[1] % cache.Hkv:
        raise ThriftError(f"q must be [B={cache.B}, H (a multiple of {cache.Hkv}), {cache.d}]")
    if q.dtype != cache.dtype:
        raise ThriftError(f"q has dtype {q.dtype}, the cache holds {cache.dtype}")
    _check_like(out, q.shape, q.dtype, "out")
    _check_like(lse, q.shape[:2], torch.float32, "lse")
    _need_cuda(q)
    B, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = attn_decode_workspace_size(B, H, cache.Hkv, cache.capacity, d, cache.blk)
    if need == 0:
        raise ThriftError("thrift_attn_decode: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_attn_decode(_ptr(q), _dt(q), B, H, cache.Hkv, d, cache.blk,
                                        cache.capacity, _ptr(cache.buf), cache.buf.numel(),
                                        _ptr(cache.lengths if seq_len is None else seq_len),
                                        _ptr(cache.kv_scale), float(topk_frac),
                                        int(sink_blocks), int(recent_blocks), int(use_scalesearch),
                                        _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(q)),
               "thrift_attn_decode")
    return out, lse


# --------------------------------------------------------------- Attn-QAT --

def qat_workspace_size(total, H, Hkv, d=128, nseq=1) -> int:
    """Bytes of the Attn-QAT workspace for ``nseq`` packed sequences of
    ``total`` tokens."""
    return int(lib().thrift_qat_workspace_size(int(total), int(nseq), H, Hkv, d))


def _qat_pack(q, k, v, cu_seqlens, max_seqlen):
    """[B,N,H,d] inputs -> packed [B*N,H,d] with uniform cu_seqlens; packed
    inputs pass through."""
    if q.dim() == 4:
        B, N = q.shape[0], q.shape[1]
        cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device=q.device)
        return (q.reshape(B * N, *q.shape[2:]), k.reshape(B * N, *k.shape[2:]),
                v.reshape(B * N, *v.shape[2:]), cu, N)
    if cu_seqlens is None or max_seqlen is None:
        raise ThriftError("packed inputs need cu_seqlens and max_seqlen")
    if cu_seqlens.dtype != torch.int32:
        raise ThriftError("cu_seqlens must be int32")
    return q, k, v, cu_seqlens, int(max_seqlen)


def thrift_qat_fwd(q, k, v, cu_seqlens=None, max_seqlen=None, blk=128, causal=True,
                   use_scalesearch=False, workspace=None):
    """Attn-QAT forward.  q [B,N,H,d] or packed [total,H,d] (with cu_seqlens,
    max_seqlen), k/v likewise with Hkv heads.  Returns (out like q in its
    dtype: the FP4 output, out_hp f32 like q: the high-precision output,
    lse f32 [H, total])."""
    _check_qkv(q, k, v, packed=q.dim() == 3)
    _need_cuda(q, k, v)
    shape = q.shape
    qp, kp, vp, cu, maxlen = _qat_pack(q, k, v, cu_seqlens, max_seqlen)
    for t in (qp, kp, vp):
        if not t.is_contiguous():
            raise ThriftError("thrift_qat_fwd: inputs must be contiguous")
    total, H, d = qp.shape
    Hkv = kp.shape[1]
    out = torch.empty_like(qp)
    out_hp = torch.empty(qp.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    need = qat_workspace_size(total, H, Hkv, d, cu.numel() - 1)
    if need == 0:
        raise ThriftError("thrift_qat_fwd: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_qat_fwd_varlen(_ptr(qp), _ptr(kp), _ptr(vp), _dt(q), _ptr(cu),
                                           cu.numel() - 1, total, maxlen, H, Hkv, d, blk, int(causal),
                                           int(use_scalesearch), _ptr(out), _ptr(out_hp), _ptr(lse),
                                           _ptr(ws), ws.numel(), _stream(q)),
               "thrift_qat_fwd_varlen")
    return out.reshape(shape), out_hp.reshape(shape), lse


def thrift_qat_bwd(q, k, v, dout, out_hp, lse, cu_seqlens=None, max_seqlen=None, blk=128,
                   causal=True, use_scalesearch=False, reuse_images=False, workspace=None):
    """Attn-QAT backward: (dq like q, dk and dv like k, all f32).
    reuse_images takes the fake-quantised images from ``workspace`` as the
    forward on the same inputs left them (an explicit workspace is then
    required)."""
    _check_qkv(q, k, v, packed=q.dim() == 3)
    total_rows = q.shape[0] * (q.shape[1] if q.dim() == 4 else 1)
    _check_like(dout, q.shape, q.dtype, "dout")
    _check_like(out_hp, q.shape, torch.float32, "out_hp")
    _check_like(lse, (q.shape[-2], total_rows), torch.float32, "lse")
    _need_cuda(q, k, v, dout, out_hp, lse)
    if reuse_images and workspace is None:
        raise ThriftError("reuse_images needs the forward's workspace")
    qshape, kshape = q.shape, k.shape
    qp, kp, vp, cu, maxlen = _qat_pack(q, k, v, cu_seqlens, max_seqlen)
    dop = dout.reshape(qp.shape)
    ohp = out_hp.reshape(qp.shape)
    for t in (qp, kp, vp, dop, ohp, lse):
        if not t.is_contiguous():
            raise ThriftError("thrift_qat_bwd: inputs must be contiguous")
    if dout.dtype != q.dtype or out_hp.dtype != torch.float32 or lse.dtype != torch.float32:
        raise ThriftError("thrift_qat_bwd: dout in the input type, out_hp and lse float32")
    total, H, d = qp.shape
    Hkv = kp.shape[1]
    dq = torch.empty(qp.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(kp.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(kp.shape, dtype=torch.float32, device=q.device)
    need = qat_workspace_size(total, H, Hkv, d, cu.numel() - 1)
    if need == 0:
        raise ThriftError("thrift_qat_bwd: unsupported shape")
    ws = workspace if workspace is not None else _ws.get(need, q.device)
    with _on(q):
        _check(lib().thrift_qat_bwd_varlen(_ptr(qp), _ptr(kp), _ptr(vp), _ptr(dop), _dt(q), _ptr(cu),
                                           cu.numel() - 1, total, maxlen, H, Hkv, d, blk, int(causal),
                                           int(use_scalesearch), int(reuse_images), _ptr(ohp),
                                           _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                           ws.numel(), _stream(q)),
               "thrift_qat_bwd_varlen")
    return dq.reshape(qshape), dk.reshape(kshape), dv.reshape(kshape)
