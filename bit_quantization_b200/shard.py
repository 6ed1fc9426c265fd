"""One attention problem split across ranks by (batch entry, kv-head group).

ThriftAttention, Metodologia step 1: the block means, pair scores and top-k
selection are taken per (sequence, head), and the NVFP4 blocks of Q, K and V
and the attention itself are per head as well.  What couples the heads and
sequences of one problem is the per-tensor FP32 scale g = amax / 2688 of Q, K
and V.  So a problem of B sequences and Hkv kv heads (each with its H / Hkv
query heads) splits into rectangular shards (a range of batch entries times a
range of kv-head groups); each rank computes its shard's three absmaxes, the
ranks agree on their elementwise maximum with one max all-reduce of 3 floats
(NCCL over NVLink on GPUs, gloo on CPU), and each rank runs the attention
call with those absmaxes.  Codes, block scales, selection and output are then
those of the whole problem on one GPU.  No data-path tensor crosses ranks.

The per-rank computations are passed in (the library's calls on GPUs), so the
same host logic is exercised by two gloo ranks on CPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch


@dataclass(frozen=True)
class Shard:
    """Batch entries [b0, b1) and kv heads [hk0, hk1) (query heads
    [hk0 * G, hk1 * G), G = H / Hkv) of one rank."""
    b0: int
    b1: int
    hk0: int
    hk1: int
    group: int  # query heads per kv head

    @property
    def h0(self):
        return self.hk0 * self.group

    @property
    def h1(self):
        return self.hk1 * self.group


def shard_of(B: int, H: int, Hkv: int, world: int, rank: int) -> Shard:
    """The rank's shard: kv-head groups split evenly when world divides Hkv,
    else batch entries when world divides B, else batch entries and kv-head
    groups both (world = wb * wh with wb | B and wh | Hkv)."""
    if H % Hkv or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard request")
    G = H // Hkv
    for wh in sorted({d for d in range(1, world + 1) if world % d == 0}, reverse=True):
        wb = world // wh
        if Hkv % wh == 0 and B % wb == 0:
            rb, rh = divmod(rank, wh)
            nb, nh = B // wb, Hkv // wh
            return Shard(rb * nb, (rb + 1) * nb, rh * nh, (rh + 1) * nh, G)
    raise ValueError(f"{world} ranks do not tile B={B} x Hkv={Hkv}")


def take(x: torch.Tensor, s: Shard, kv: bool) -> torch.Tensor:
    """The shard's part of a [B, N, heads, d] tensor (kv: heads are kv heads),
    contiguous."""
    h0, h1 = (s.hk0, s.hk1) if kv else (s.h0, s.h1)
    return x[s.b0:s.b1, :, h0:h1].contiguous()


def agree_absmax(amax: torch.Tensor, world: int) -> torch.Tensor:
    """Elementwise maximum of the ranks' [3] absmax tensors, in place (one
    all-reduce of 3 floats in the process group)."""
    if world > 1:
        torch.distributed.all_reduce(amax, op=torch.distributed.ReduceOp.MAX)
    return amax


def sharded_step(q_s, k_s, v_s, world: int,
                 absmax: Callable[..., torch.Tensor],
                 attend: Callable[..., object]):
    """One attention step on this rank's shard: local absmaxes, the max
    all-reduce, then the attention with the agreed absmaxes.  `absmax(q, k,
    v)` returns a float32 [3] tensor; `attend(q, k, v, amax)` runs the
    attention and returns its result."""
    amax = absmax(q_s, k_s, v_s)
    agree_absmax(amax, world)
    return attend(q_s, k_s, v_s, amax)
