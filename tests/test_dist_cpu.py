"""The benchmark's multi-rank logic (bit_quantization_b200/dist.py) with two
gloo ranks on CPU: the process group, the barrier, the maximum over ranks of
the elapsed times, the sum over ranks of the work, the whole-job rate, one
problem per rank (distinct seeds), and the CPU reference arm running on rank
0 only."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from bit_quantization_b200 import dist, synth
    w_, r_, _ = dist.setup("gloo", timeout_s=30)
    dist.barrier(w_)
    elapsed = [10.0 * (r_ + 1), 5.0 - r_]          # this rank's timings (ms)
    work = [1.0e12 * (r_ + 1)]                      # this rank's flops
    mx = dist.max_over_ranks(elapsed, w_)
    sm = dist.sum_over_ranks(work, w_)
    seed = dist.rank_seed(synth.TINY.seed, r_)
    q = synth.make_attn_inputs(synth.TINY, seed=seed)["q"]
    res = {"world": w_, "rank": r_, "max": mx, "sum": sm, "seed": seed,
           "rate": dist.whole_job_rate(sm[0], mx[0]), "q_sum": float(q.float().sum())}
    dist.barrier(w_)
    dist.teardown(w_)
    with open(os.path.join(outdir, f"rank{r_}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["world"] == world and d["rank"] == r
        assert d["max"] == [20.0, 5.0]              # maximum over ranks, element-wise
        assert d["sum"] == [3.0e12]                 # work of both ranks
        assert d["rate"] == pytest.approx(3.0e12 / 20e-3)
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["q_sum"] != res[1]["q_sum"]       # each rank draws its own problem


def test_single_rank_needs_no_process_group(monkeypatch):
    from bit_quantization_b200 import dist
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert dist.setup("gloo") == (1, 0, 0)
    assert dist.max_over_ranks([3.0, 1.0], 1) == [3.0, 1.0]
    assert dist.sum_over_ranks([2.0], 1) == [2.0]
    dist.barrier(1)
    dist.teardown(1)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    from bit_quantization_b200 import synth
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, ref_units = 1, 0, 1

    assert bench.run_reference(Args(), synth.TINY) == 0
    assert capsys.readouterr().out == ""
