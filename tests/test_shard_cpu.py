"""One attention problem split across two gloo ranks on CPU by kv-head group
(bit_quantization_b200/shard.py; ThriftAttention Metodologia step 1: every
step but the per-tensor scales is per (sequence, head)).  Each rank takes its
shard of the inputs, computes the shard's three absmaxes, the ranks agree on
their maximum with one all-reduce, and the rank's attention runs under the
agreed scales.  The per-rank computations are the oracle's here (the same
host logic drives the library's calls on GPUs); the shards' codes, block
scales, selection and outputs must equal the slices of the one-rank run bit
for bit."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

B, H, HKV, N, D, BLK = 2, 4, 2, 192, 64, 64
FLAGS = dict(causal=True, frac=0.25, ss=True, had=True)


def _workload():
    from bit_quantization_b200 import synth
    return synth.AttnWorkload("shard", B, H, HKV, N, D, torch.bfloat16, FLAGS["causal"], BLK,
                              FLAGS["frac"], FLAGS["ss"], FLAGS["had"], k_offset_std=3.0, seed=4)


def _oracle_attend(orc, q, k, v, g):
    from bit_quantization_b200 import synth
    b, n, hs, d = q.shape
    cu = np.arange(b + 1, dtype=np.int32) * n
    qp, kp, vp = (synth.as_u16(t.reshape(b * n, -1, d)) for t in (q, k, v))
    r = orc.thrift_attn(qp, kp, vp, 1, cu, BLK, FLAGS["causal"], FLAGS["frac"],
                        use_ss=FLAGS["ss"], use_had=FLAGS["had"], g=g)
    codes, scales, _, _ = orc.nvfp4_quantize(qp.reshape(-1, d), 1, use_ss=FLAGS["ss"],
                                             use_had=FLAGS["had"], g=g[0])
    return r, codes, scales


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import oracle as orc
    from bit_quantization_b200 import dist, shard, synth
    w_, r_, _ = dist.setup("gloo", timeout_s=60)
    inp = synth.make_attn_inputs(_workload())
    s = shard.shard_of(B, H, HKV, w_, r_)
    q_s, k_s, v_s = (shard.take(inp[n], s, kv=n != "q") for n in ("q", "k", "v"))

    def absmax(q, k, v):
        return torch.tensor([orc.tensor_absmax(synth.as_u16(q), 1, hadamard=FLAGS["had"]),
                             orc.tensor_absmax(synth.as_u16(k), 1, hadamard=FLAGS["had"]),
                             orc.tensor_absmax(synth.as_u16(v), 1)], dtype=torch.float32)

    def attend(q, k, v, amax):
        g = [orc.scale_from_absmax(float(a)) for a in amax]
        return g, _oracle_attend(orc, q, k, v, g)

    g, (r, codes, scales) = shard.sharded_step(q_s, k_s, v_s, w_, absmax, attend)
    np.savez(os.path.join(outdir, f"rank{r_}.npz"), out=r["out"], out64=r["out64"],
             mask=r["mask"], codes=codes, scales=scales, g=np.array(g, np.float32))
    with open(os.path.join(outdir, f"rank{r_}.json"), "w") as f:
        json.dump({"shard": [s.b0, s.b1, s.hk0, s.hk1]}, f)
    dist.barrier(w_)
    dist.teardown(w_)


def test_two_ranks_match_one(tmp_path, orc):
    from bit_quantization_b200 import synth
    world, port = 2, None
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    inp = synth.make_attn_inputs(_workload())
    cu = np.arange(B + 1, dtype=np.int32) * N
    qp, kp, vp = (synth.as_u16(inp[n].reshape(B * N, -1, D)) for n in ("q", "k", "v"))
    full = orc.thrift_attn(qp, kp, vp, 1, cu, BLK, FLAGS["causal"], FLAGS["frac"],
                           use_ss=FLAGS["ss"], use_had=FLAGS["had"])
    fcodes, fscales, _, _ = orc.nvfp4_quantize(qp.reshape(-1, D), 1, use_ss=FLAGS["ss"],
                                               use_had=FLAGS["had"])
    nb = (N + BLK - 1) // BLK
    fmask = full["mask"].reshape(B, H, nb, nb)
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npz")
        b0, b1, hk0, hk1 = json.load(open(tmp_path / f"rank{r}.json"))["shard"]
        h0, h1 = hk0 * (H // HKV), hk1 * (H // HKV)
        hs = h1 - h0
        assert np.array_equal(got["g"], np.array(full["g"], np.float32))
        assert np.array_equal(got["mask"].reshape(b1 - b0, hs, nb, nb), fmask[b0:b1, h0:h1])
        fo = full["out"].reshape(B, N, H, D)[b0:b1, :, h0:h1]
        assert np.array_equal(got["out"].reshape(fo.shape), fo)
        f64 = full["out64"].reshape(B, N, H, D)[b0:b1, :, h0:h1]
        assert np.array_equal(got["out64"].reshape(f64.shape), f64)
        fc = fcodes.reshape(B, N, H, D // 2)[b0:b1, :, h0:h1]
        assert np.array_equal(got["codes"].reshape(fc.shape), fc)
        fs = fscales.reshape(B, N, H, D // 16)[b0:b1, :, h0:h1]
        assert np.array_equal(got["scales"].reshape(fs.shape), fs)


@pytest.mark.parametrize("B_,H_,Hkv_,world", [(1, 32, 8, 8), (2, 32, 32, 4), (4, 32, 8, 2),
                                              (4, 32, 2, 8), (3, 16, 16, 16)])
def test_shards_tile_the_problem(B_, H_, Hkv_, world):
    from bit_quantization_b200 import shard
    seen = np.zeros((B_, H_), int)
    for r in range(world):
        s = shard.shard_of(B_, H_, Hkv_, world, r)
        assert s.h1 - s.h0 == (s.hk1 - s.hk0) * (H_ // Hkv_)
        seen[s.b0:s.b1, s.h0:s.h1] += 1
    assert np.all(seen == 1)  # every (batch entry, query head) on exactly one rank


def test_untileable_world_is_rejected():
    from bit_quantization_b200 import shard
    with pytest.raises(ValueError):
        shard.shard_of(1, 32, 8, 3, 0)
