"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and nothing else: it holds none of the
quantisation, selection or attention arithmetic.  Both the CUDA path and the
CPU oracle consume exactly the tensors produced here.

Recipe (stand-in for the long-context LLM attention inputs the pages evaluate
on; their datasets and model weights are not used):
  * one ``torch.Generator`` seeded with ``seed``;
  * draw order: sequence lengths -> Q -> K -> V -> K channel offsets ->
    outlier channels (the last two only when asked for);
  * values are fp32 ``randn`` cast once, round-to-nearest, to the 16-bit type;
  * K channel offsets: mu ~ 3 * randn(Hkv, d), added to K in fp32 before the
    cast and shared by every batch entry and token;
  * outlier channels (quantiser workload): 4 channels from ``randperm(cols)``
    multiplied by 20 before the cast;
  * decode (one query token per sequence against a cache): draw order
    cached lengths (uniform on [lo, hi] unless given) -> K cache -> V cache
    -> K channel offsets -> the step's query tokens; the cache tensors
    [B, capacity, Hkv, d] are drawn whole, so tokens past a sequence's
    length hold random values that a correct decode never reads.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class AttnWorkload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int            # tokens per sequence (max length for varlen)
    d: int
    dtype: torch.dtype
    causal: bool
    blk: int
    topk_frac: float
    use_scalesearch: bool
    use_hadamard: bool
    k_offset_std: float = 0.0
    varlen: Optional[dict] = None   # {"nseq": n, "lo": a, "hi": b}
    seed: int = 0


@dataclass
class QuantWorkload:
    name: str
    rows: int
    cols: int
    dtype: torch.dtype
    n_outlier_channels: int
    outlier_scale: float
    seed: int = 0


@dataclass
class DecodeWorkload:
    name: str
    B: int
    H: int
    Hkv: int
    capacity: int     # cache slots per sequence
    lo: int           # cached lengths uniform on [lo, hi]
    hi: int
    d: int
    dtype: torch.dtype
    topk_frac: float
    use_scalesearch: bool
    k_offset_std: float = 3.0
    sink_blocks: int = 0
    recent_blocks: int = 0
    seed: int = 0


TINY = AttnWorkload("tiny_b1h1n256d64_fp16", 1, 1, 1, 256, 64, torch.float16, False, 64, 0.25,
                    False, False)
QUANT = QuantWorkload("quant_65536x128_fp16_4outliers", 65536, 128, torch.float16, 4, 20.0)
C_B2H32N8K = AttnWorkload("b2h32n8192d128_bf16_noncausal_top10", 2, 32, 32, 8192, 128,
                          torch.bfloat16, False, 128, 0.10, False, False, k_offset_std=3.0)
C_GQA32K = AttnWorkload("b1h32hkv8n32768d128_bf16_causal_had_ss_top5", 1, 32, 8, 32768, 128,
                        torch.bfloat16, True, 128, 0.05, True, True, k_offset_std=3.0)
C_VARLEN = AttnWorkload("varlen16_1k16k_h16d128_bf16_causal_had_ss", 16, 16, 16, 16384, 128,
                        torch.bfloat16, True, 128, 0.05, True, True, k_offset_std=3.0,
                        varlen={"nseq": 16, "lo": 1024, "hi": 16384})


# Llama-3.1-8B attention shape (32 query heads, 8 kv heads, d = 128) at the
# 131k context the pages quote decode at.
# 131072 tokens cached per sequence, room for one more tile of new tokens.
C_DECODE131K = DecodeWorkload("decode_b4h32hkv8_ctx131072_bf16_top10", 4, 32, 8, 131072 + 128,
                              131072, 131072, 128, torch.bfloat16, 0.10, False)


@dataclass
class QatWorkload:
    name: str
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    dtype: torch.dtype
    causal: bool
    blk: int
    use_scalesearch: bool
    k_offset_std: float = 3.0
    seed: int = 0


# Attn-QAT training step (forward + backward) at the Llama-3.1-8B attention
# shape and a 4k training context; the pages give no training shapes.
C_QAT4K = QatWorkload("qat_b1h32hkv8n4096d128_bf16_causal", 1, 32, 8, 4096, 128, torch.bfloat16,
                      True, 128, False)


def varlen_lengths(gen: torch.Generator, nseq: int, lo: int, hi: int):
    """Integer lengths uniform on [lo, hi] (inclusive)."""
    return torch.randint(lo, hi + 1, (nseq,), generator=gen).tolist()


def make_attn_inputs(w: AttnWorkload, seed: Optional[int] = None, lengths=None):
    """Returns dict(q, k, v, cu_seqlens (int32, CPU), lengths).

    Non-varlen: q [B,N,H,d], k/v [B,N,Hkv,d].  Varlen: q [total,H,d],
    k/v [total,Hkv,d] packed, cu_seqlens [nseq+1].  All on CPU."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    if w.varlen is not None:
        if lengths is None:
            lengths = varlen_lengths(gen, w.varlen["nseq"], w.varlen["lo"], w.varlen["hi"])
        total = int(sum(lengths))
        qs, ks = (total, w.H, w.d), (total, w.Hkv, w.d)
    else:
        lengths = [w.N] * w.B
        qs, ks = (w.B, w.N, w.H, w.d), (w.B, w.N, w.Hkv, w.d)
    q = torch.randn(qs, generator=gen, dtype=torch.float32)
    k = torch.randn(ks, generator=gen, dtype=torch.float32)
    v = torch.randn(ks, generator=gen, dtype=torch.float32)
    if w.k_offset_std:
        mu = w.k_offset_std * torch.randn((w.Hkv, w.d), generator=gen, dtype=torch.float32)
        k += mu
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    return {"q": q.to(w.dtype), "k": k.to(w.dtype), "v": v.to(w.dtype), "cu_seqlens": cu,
            "lengths": list(lengths)}


def make_decode_inputs(w: DecodeWorkload, seed: Optional[int] = None, lengths=None,
                       device="cpu"):
    """Returns dict(q [B,H,d], k, v [B,capacity,Hkv,d], lengths (list)).
    ``device`` = "cuda" draws on the GPU (for caches too large to move)."""
    gen = torch.Generator(device=device).manual_seed(w.seed if seed is None else seed)
    if lengths is None:
        lengths = torch.randint(w.lo, w.hi + 1, (w.B,), generator=gen, device=device).tolist()
    ks = (w.B, w.capacity, w.Hkv, w.d)
    k = torch.randn(ks, generator=gen, dtype=torch.float32, device=device)
    v = torch.randn(ks, generator=gen, dtype=torch.float32, device=device).to(w.dtype)
    if w.k_offset_std:
        mu = w.k_offset_std * torch.randn((w.Hkv, w.d), generator=gen, dtype=torch.float32,
                                          device=device)
        k += mu
    k = k.to(w.dtype)
    q = torch.randn((w.B, w.H, w.d), generator=gen, dtype=torch.float32, device=device)
    return {"q": q.to(w.dtype), "k": k, "v": v, "lengths": list(lengths)}


def make_quant_input(w: QuantWorkload, seed: Optional[int] = None):
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    x = torch.randn((w.rows, w.cols), generator=gen, dtype=torch.float32)
    if w.n_outlier_channels:
        ch = torch.randperm(w.cols, generator=gen)[: w.n_outlier_channels]
        x[:, ch] *= w.outlier_scale
    return x.to(w.dtype)


def randn16(shape, dtype, seed, scale=1.0):
    """Plain seeded N(0, scale^2) tensor of a 16-bit type (tests)."""
    gen = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(shape, generator=gen, dtype=torch.float32)).to(dtype)


def as_u16(t: torch.Tensor):
    """Bit pattern of a 16-bit CPU tensor as a numpy uint16 array."""
    import numpy as np
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def dtype_code(dtype: torch.dtype) -> int:
    return {torch.float16: 0, torch.bfloat16: 1}[dtype]


def make_qat_inputs(w: QatWorkload, seed: Optional[int] = None, lengths=None, device="cpu"):
    """Returns dict(q [total,H,d], k, v [total,Hkv,d], dout [total,H,d],
    cu_seqlens int32 [nseq+1], lengths).  Draw order: lengths (given, else
    B x N) -> Q -> K -> V -> K channel offsets -> dO (the output gradient,
    N(0,1))."""
    gen = torch.Generator(device=device).manual_seed(w.seed if seed is None else seed)
    if lengths is None:
        lengths = [w.N] * w.B
    total = int(sum(lengths))
    f32 = torch.float32
    q = torch.randn((total, w.H, w.d), generator=gen, dtype=f32, device=device)
    k = torch.randn((total, w.Hkv, w.d), generator=gen, dtype=f32, device=device)
    v = torch.randn((total, w.Hkv, w.d), generator=gen, dtype=f32, device=device)
    if w.k_offset_std:
        k += w.k_offset_std * torch.randn((w.Hkv, w.d), generator=gen, dtype=f32, device=device)
    dout = torch.randn((total, w.H, w.d), generator=gen, dtype=f32, device=device)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    return {"q": q.to(w.dtype), "k": k.to(w.dtype), "v": v.to(w.dtype), "dout": dout.to(w.dtype),
            "cu_seqlens": cu, "lengths": list(lengths)}
