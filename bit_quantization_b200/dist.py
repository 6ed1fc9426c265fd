"""Multi-rank plumbing of the benchmark: one process per GPU, each on its
own problem (weak scaling: independent batches, sequences or heads, so
nothing crosses ranks on the data path).  Only timings and work counts cross
ranks, through the process group: the elapsed time of a run is the maximum
over ranks, the work done is the sum over ranks.  NCCL on GPUs; gloo for the
CPU tests of the same logic."""
from __future__ import annotations

import datetime
import os

import torch


def env():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def setup(backend: str = "nccl", timeout_s: float = 120.0):
    """Joins the process group when there is more than one rank (the
    launcher's MASTER_ADDR / MASTER_PORT); returns env()."""
    world, rank, local = env()
    if world > 1:
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend,
                                             timeout=datetime.timedelta(seconds=timeout_s))
    return world, rank, local


def _device():
    if torch.distributed.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def _reduce(values, op, world: int):
    if world == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=_device())
    torch.distributed.all_reduce(t, op=op)
    return [float(x) for x in t.cpu()]


def max_over_ranks(values, world: int):
    """Element-wise maximum over ranks (elapsed times)."""
    return _reduce(values, torch.distributed.ReduceOp.MAX if world > 1 else None, world)


def sum_over_ranks(values, world: int):
    """Element-wise sum over ranks (work done)."""
    return _reduce(values, torch.distributed.ReduceOp.SUM if world > 1 else None, world)


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic problem: every rank draws its own inputs."""
    return base + rank


def whole_job_rate(total_units: float, max_ms: float) -> float:
    """Units of all ranks per second of the slowest rank."""
    return total_units / (max_ms * 1e-3)


def teardown(world: int):
    if world > 1:
        torch.distributed.destroy_process_group()
