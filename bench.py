#!/usr/bin/env python
"""Benchmark of the NVFP4 / selective-FP16 attention forward on B200.

One step = one thrift_attn_fwd call over one batch of the workload: tensor
absmax, Q/K/V NVFP4 quantisation, block-mean top-k selection and the mixed
NVFP4/FP16 attention kernel.  Prints one JSON line (rank 0).

Default workload: B=2, H=32, N=8192, d=128, bf16, non-causal, 128x128 blocks,
10% FP16 pairs, K with per-channel offsets N(0, 3).  Its inputs (3 x 134 MB)
exceed L2, so no flush is needed between steps.

The line also carries "decode": one decode step of the double-cache decode
path (Llama-3.1-8B attention shape, B=4, 131072 cached tokens, 10% FP16
tiles): append the step's token, then attend; its kernel against HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference   # the CPU oracle on a bounded sample
Multi-GPU (weak scaling, independent problems per rank, no collective on the
data path): launched by torch.distributed.run, one rank per GPU.
"""
import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_quantization_b200 import dist, synth  # noqa: E402

WORKLOADS = {
    "b2h32n8192": synth.C_B2H32N8K,
    "gqa32k": synth.C_GQA32K,
    "tiny": synth.TINY,
}

METRIC = "NVFP4 attention fwd TFLOPS (whole step: quantise + select + attention)"
UNIT = "TFLOP/s"
KERNELS_PER_STEP = 9  # 3 absmax, 2 Q/K images (with the block means), 1 V image, 1 scores, 1 top-k, 1 attention


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# DRAM traffic of one attention launch measured by ncu (read + write bytes)
# for the attention source with this hash; reported only while the source is
# unchanged since the capture.
ATTN_TRAFFIC = {"src_sha16": "aed717716c579cc9", "workload": "b2h32n8192d128_bf16_noncausal_top10",
                "bytes": 396740352 + 123007744}


def attn_traffic(w):
    import hashlib
    path = os.path.join(ROOT, "bit_quantization_b200", "csrc", "attn.cuh")
    sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    if sha == ATTN_TRAFFIC["src_sha16"] and w.name == ATTN_TRAFFIC["workload"]:
        return ATTN_TRAFFIC["bytes"]
    return None


# DRAM traffic per step of the three Attn-QAT attention kernels (forward,
# key-tile and query-tile backward) from the ncu launch list of the QAT source
# with this hash; reported only while the source is unchanged.
QAT_TRAFFIC = {"src_sha16": "932e539dcdf5cdaa", "workload": "qat_b1h32hkv8n4096d128_bf16_causal",
               "bytes": int((99.2 + 90.2 + 111.9) * 1e6)}


def qat_traffic(w):
    import hashlib
    path = os.path.join(ROOT, "bit_quantization_b200", "csrc", "qat.cuh")
    sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    if sha == QAT_TRAFFIC["src_sha16"] and w.name == QAT_TRAFFIC["workload"]:
        return QAT_TRAFFIC["bytes"]
    return None


XU_OPS_PER_CLK_PER_SM = 16   # MUFU lanes per SM (4 per sub-partition)
# MUFU operations per score element: one exp2, plus one exp2 and one log2 per
# 16-key block for the block scale (the E2M1 / 16-bit converts do not use
# this pipe: an instruction-class count of each convert shows none there)
XU_OPS_PER_ELEMENT = 1.125


def pair_flops(mask, w, lengths):
    """Algorithmic FLOPs (4*d per unmasked score element) split by path."""
    blk, d = w.blk, w.d
    f4 = f16 = 0.0
    for b, L in enumerate(lengths):
        nb = (L + blk - 1) // blk
        for i in range(nb):
            r0, r1 = i * blk, min(L, (i + 1) * blk)
            for j in range(nb if not w.causal else i + 1):
                c0, c1 = j * blk, min(L, (j + 1) * blk)
                if w.causal:
                    rows = np.arange(r0, r1)
                    cnt = float(np.clip(np.minimum(rows + 1, c1) - c0, 0, None).sum())
                else:
                    cnt = float((r1 - r0) * (c1 - c0))
                sel = mask[b, :, i, j]
                n16 = float(sel.sum())
                f16 += 4 * d * cnt * n16
                f4 += 4 * d * cnt * (w.H - n16)
    return f4, f16


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.proc = None
        self.dev_id = None
        try:
            uuid = torch.cuda.get_device_properties(dev).uuid
            self.dev_id = "GPU-" + str(uuid)
        except Exception:
            self.dev_id = str(dev.index or 0)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.dev_id, f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_sample(w, nunits, nthreads, inp=None):
    """The CPU oracle on a bounded sample of the workload: one head of batch
    entry 0 (full sequence length), `nunits` evenly spread query blocks.
    Returns (seconds, algorithmic flops of the sampled rows, description)."""
    import oracle
    if inp is None:
        inp = synth.make_attn_inputs(w)
    N, d, blk = w.N, w.d, w.blk
    q = inp["q"][0, :, 0:1].contiguous()
    k = inp["k"][0, :, 0:1].contiguous()
    v = inp["v"][0, :, 0:1].contiguous()
    cu = np.array([0, N], np.int32)
    nb = (N + blk - 1) // blk
    blocks = np.unique(np.linspace(0, nb - 1, nunits).round().astype(int))
    units = np.array([[0, 0, i] for i in blocks], np.int32)
    t0 = time.perf_counter()
    oracle.thrift_attn(synth.as_u16(q), synth.as_u16(k), synth.as_u16(v), synth.dtype_code(w.dtype),
                       cu, blk, w.causal, w.topk_frac, use_ss=w.use_scalesearch,
                       use_had=w.use_hadamard, units=units, nthreads=nthreads)
    dt = time.perf_counter() - t0
    fl = 0.0
    for i in blocks:
        rows = np.arange(i * blk, min(N, (i + 1) * blk))
        cnt = (rows + 1).sum() if w.causal else len(rows) * N
        fl += 4.0 * d * cnt
    desc = (f"1 of {w.B * w.H} heads (batch 0, head 0, full N={N}), {len(blocks)} of {nb} query "
            f"blocks; includes that head's quantisation and selection")
    return dt, fl, desc


def run_reference(args, w):
    world, rank, _ = dist.env()
    if rank != 0:
        return 0  # the CPU reference runs once, on rank 0
    cores = os.cpu_count() or 1
    inp = synth.make_attn_inputs(w)
    # Size the sample so the whole run stays within about two minutes.
    dt0, _, _ = oracle_sample(w, 4, cores, inp)
    budget = min(4.0, 120.0 / (args.steps + args.warmup))
    units = int(max(1, min(args.ref_units, 4 * budget / max(dt0, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(w, units, cores, inp)
    times, fl, desc = [], 0.0, ""
    for _ in range(args.steps):
        dt, fl, desc = oracle_sample(w, units, cores, inp)
        times.append(dt)
    t = sum(times)
    val = fl * args.steps / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "d": w.d,
            "dtype": str(w.dtype).replace("torch.", ""), "causal": w.causal, "blk": w.blk,
            "topk_frac": w.topk_frac, "scalesearch": w.use_scalesearch,
            "hadamard": w.use_hadamard, "k_offset_std": w.k_offset_std,
            "l2": "inputs larger than L2 (no flush)", "parallelism": "independent problems per GPU"}


def quantizer_line(dev, peaks):
    """Quantiser-only workload (65536 x 128 fp16 with 4 outlier channels):
    GB/s of algorithmic bytes (2 B read + 0.5625 B written per element).
    Twelve rotating input copies (> L2); the calls are captured in one CUDA
    graph so host-side launch gaps do not enter the timing."""
    from bit_quantization_b200 import ops
    x0 = synth.make_quant_input(synth.QUANT).to(dev)
    xs = [x0.clone() for _ in range(12)]
    rows, cols = x0.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    ws = torch.zeros(ops.lib().nvfp4_quantize_workspace_size(), dtype=torch.uint8, device=dev)
    res = {}
    algo = rows * cols * (2 + 0.5 + 0.0625)
    n = 120
    gts = ops.nvfp4_quantize(x0, False, False, None, codes, scales, ws)[2].clone()  # g of x0
    for ss, given in ((False, False), (True, False), (False, True)):
        ts = gts if given else None
        for i in range(6):
            ops.nvfp4_quantize(xs[i % 12], ss, False, ts, codes, scales, ws)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        with torch.cuda.graph(g, stream=side):
            for i in range(n):
                ops.nvfp4_quantize(xs[i % 12], ss, False, ts, codes, scales, ws)
        g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(3):
            g.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / (3 * n)
        gbs = algo / (ms * 1e-3) / 1e9
        key = ("scalesearch_on" if ss else "scalesearch_off") + ("_scale_given" if given else "")
        res[key] = {"us_per_call": 1e3 * ms, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
                    "kernels_per_call": 1}
        del g
    res["workload"] = synth.QUANT.name
    res["algorithmic_bytes"] = algo
    res["timing"] = "CUDA graph of 120 calls, 12 rotating inputs (201 MB > L2)"
    return res


def quantizer_only(args):
    """A few plain (not graph-captured) quantiser calls on the quantiser
    workload, ScaleSearch off then on; prints their event-timed durations."""
    from bit_quantization_b200 import ops
    dev = torch.device("cuda", 0)
    x = synth.make_quant_input(synth.QUANT).to(dev)
    res = {}
    for ss in (False, True):
        times = []
        for _ in range(args.warmup + args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ops.nvfp4_quantize(x, ss)
            e1.record()
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
        res["ss_on" if ss else "ss_off"] = 1e3 * min(times[args.warmup:])
    print(json.dumps({"mode": "quantizer", "workload": synth.QUANT.name, "us_min": res}))
    return 0


DECODE_KERNELS_PER_STEP = 7  # append (2), query images (absmax fused), scores, top-k, decode, merge

# DRAM traffic per algorithmic byte of the decode kernel, measured by ncu on
# the 32768-token case of the decode workload (the traffic scales with the
# tiles read); reported only while the decode source is unchanged since.
DECODE_TRAFFIC = {"src_sha16": "a565554521ecf748", "bytes_per_algorithmic_byte": 344.61 / 338.72,
                  "captured_on": "decode workload with 32768 cached tokens"}


def decode_setup(ops, dev, w, context=None):
    """The decode workload's cache filled on the GPU: (cache, q, k_new,
    v_new, L0, workspace, kv scales).  ``context`` overrides the cached
    length (profiling on a smaller case)."""
    if context is not None:
        w = dataclasses.replace(w, capacity=context + 128, lo=context, hi=context)
    inp = synth.make_decode_inputs(w, device=dev)
    q, k, v = inp["q"], inp["k"], inp["v"]
    L0 = inp["lengths"][0]
    # the cache's per-tensor scales: the library's own quantiser over the
    # cached tokens (g = amax / 2688, reading R1)
    kv = torch.stack([ops.nvfp4_quantize(k[:, :L0].reshape(-1, w.d))[2].reshape(()),
                      ops.nvfp4_quantize(v[:, :L0].reshape(-1, w.d))[2].reshape(())])
    cache = ops.DoubleKVCache(w.B, w.Hkv, w.capacity, kv, dtype=w.dtype)
    for t0 in range(0, L0, 32768):
        t1 = min(L0, t0 + 32768)
        cache.append(k[:, t0:t1].contiguous(), v[:, t0:t1].contiguous())
    k_new = k[:, L0:L0 + 1].contiguous()
    v_new = v[:, L0:L0 + 1].contiguous()
    del k, v, inp
    ws = torch.empty(ops.attn_decode_workspace_size(w.B, w.H, w.Hkv, w.capacity), dtype=torch.uint8,
                     device=dev)
    return w, cache, q, k_new, v_new, L0, ws


def decode_traffic(kv_bytes):
    import hashlib
    with open(os.path.join(ROOT, "bit_quantization_b200", "csrc", "decode.cuh"), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if sha != DECODE_TRAFFIC["src_sha16"]:
        return None
    return kv_bytes * DECODE_TRAFFIC["bytes_per_algorithmic_byte"]


def decode_tiles(ops, w, ws, L0):
    """Key tiles the last decode step read, from the selection it left in
    the workspace: per (sequence, kv head), every tile some query head took
    in NVFP4 (K4 + V4 = 18432 B) and every tile some head took in FP16
    (K16 + V16 = 65536 B).  Returns (tiles NVFP4, tiles FP16, bytes)."""
    nbcap = (w.capacity + 127) // 128
    mo = ops.attn_decode_mask_offset(w.B, w.H, w.Hkv, w.capacity)
    mask = ws[mo:mo + w.B * w.H * nbcap].view(w.B, w.Hkv, w.H // w.Hkv, nbcap).bool()
    mask = mask[..., :(L0 + 1 + 127) // 128]
    t16 = int(mask.any(dim=2).sum())
    t4 = int((~mask.all(dim=2)).sum())
    return t4, t16, t4 * 18432 + t16 * 65536


def decode_line(ops, dev, peaks, steps=50, warmup=5):
    """One decode step of the decode workload (Llama-3.1-8B attention shape,
    131072 cached tokens per sequence): append the step's token to every
    sequence's double cache, then attend.  The cached length is reset before
    each step, so every step appends at the same position and attends over
    131073 tokens."""
    w, cache, q, k_new, v_new, L0, ws = decode_setup(ops, dev, synth.C_DECODE131K)
    # the serving loop's own length bookkeeping: every step writes its token
    # at position L0 and attends over L0 + 1 tokens
    at = torch.full((w.B,), L0, dtype=torch.int32, device=dev)
    ones = torch.ones(w.B, dtype=torch.int32, device=dev)
    lens = at + ones
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H), dtype=torch.float32, device=dev)

    def step():
        cache.append(k_new, v_new, n_new=ones, cache_len=at)
        ops.thrift_attn_decode(q, cache, topk_frac=w.topk_frac, out=out, lse=lse, workspace=ws,
                               seq_len=lens)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out in the decode warm-up")
    ops.kernel_timer_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize(dev)
    kms, nk = ops.kernel_timer_read()
    ops.kernel_timer_enable(False)
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out in the decode loop")
    step_us = 1e3 * e0.elapsed_time(e1) / steps
    k_us = 1e3 * kms / max(nk, 1)
    # the same step replayed from a CUDA graph (one capture, no per-kernel
    # launch cost), the way a serving loop runs a fixed-shape decode step
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    graph_us = 1e3 * e0.elapsed_time(e1) / steps
    del graph
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out in the decode graph")
    t4, t16, kv_bytes = decode_tiles(ops, w, ws, L0)
    achieved = kv_bytes / (k_us * 1e-6) / 1e9
    hbm = peaks["hbm_gbs"]
    return {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "d": w.d,
            "cached_tokens": L0, "attended_tokens": L0 + 1, "topk_frac": w.topk_frac,
            "us_per_step": step_us, "us_per_step_graph": graph_us, "steps": steps,
            "step": "append one token per sequence to the FP4 + 16-bit cache, then attend",
            "kernel_us": k_us, "tiles_nvfp4": t4, "tiles_fp16": t16,
            "roofline": {"bound": "hbm", "kernel": "attn_decode_kernel", "achieved": achieved,
                         "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": decode_traffic(kv_bytes), "algorithmic_bytes": kv_bytes,
                         "traffic_note": "ncu DRAM bytes of a 32768-token launch per algorithmic "
                                         "byte, times this launch's algorithmic bytes"},
            "kernels_per_step": DECODE_KERNELS_PER_STEP}


def decode_only(args):
    """A few decode steps (profiling aid); ``--decode-context`` sets the
    cached length."""
    from bit_quantization_b200 import ops
    dev = torch.device("cuda", 0)
    w, cache, q, k_new, v_new, L0, ws = decode_setup(ops, dev, synth.C_DECODE131K,
                                                   args.decode_context)
    at = torch.full((w.B,), L0, dtype=torch.int32, device=dev)
    ones = torch.ones(w.B, dtype=torch.int32, device=dev)
    lens = at + ones
    times = []
    for _ in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        cache.append(k_new, v_new, n_new=ones, cache_len=at)
        ops.thrift_attn_decode(q, cache, topk_frac=w.topk_frac, workspace=ws, seq_len=lens)
        e1.record()
        torch.cuda.synchronize(dev)
        times.append(1e3 * e0.elapsed_time(e1))
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out")
    t4, t16, kv_bytes = decode_tiles(ops, w, ws, L0)
    print(json.dumps({"mode": "decode", "workload": w.name, "cached_tokens": L0,
                      "us_min": min(times[args.warmup:]), "tiles_nvfp4": t4, "tiles_fp16": t16,
                      "algorithmic_bytes": kv_bytes}))
    return 0


def qat_setup(ops, dev, w):
    inp = synth.make_qat_inputs(w, device=dev)
    q, k, v, dout = (inp[n] for n in ("q", "k", "v", "dout"))
    cu = inp["cu_seqlens"].to(dev)
    ws = torch.empty(ops.qat_workspace_size(q.shape[0], w.H, w.Hkv, w.d), dtype=torch.uint8,
                     device=dev)
    return inp, q, k, v, dout, cu, ws


def qat_flops(w, lengths):
    """Algorithmic FLOPs of one Attn-QAT step: the forward's S, P^V and PV and
    the backward's dP, dV, dK and dQ, 2 d flops per visible (query, key)
    pair each."""
    pairs = sum(L * (L + 1) // 2 if w.causal else L * L for L in lengths) * w.H
    return 7 * 2 * pairs * w.d, pairs


# forward: 3 tensor absmax, 3 image kernels, the attention forward; backward
# (images reused): D, the key-tile and the query-tile gradient kernels
QAT_KERNELS_PER_STEP = 10


def qat_line(ops, dev, peaks, peak_src, args, steps=20, warmup=3):
    """Attn-QAT training step (forward + backward) of the QAT workload: the
    forward quantises Q, K, V and writes O, O', lse; the backward reuses the
    forward's images and returns dQ, dK, dV."""
    w = synth.C_QAT4K
    inp, q, k, v, dout, cu, ws = qat_setup(ops, dev, w)
    N = w.N

    def fwd():
        return ops.thrift_qat_fwd(q, k, v, cu, N, blk=w.blk, causal=w.causal,
                                  use_scalesearch=w.use_scalesearch, workspace=ws)

    out, out_hp, lse = fwd()

    def bwd():
        return ops.thrift_qat_bwd(q, k, v, dout, out_hp, lse, cu, N, blk=w.blk, causal=w.causal,
                                  use_scalesearch=w.use_scalesearch, reuse_images=True,
                                  workspace=ws)

    for _ in range(warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out in the QAT warm-up")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps + 1)]
    ev[0].record()
    for i in range(steps):
        fwd()
        ev[2 * i + 1].record()
        bwd()
        ev[2 * i + 2].record()
    torch.cuda.synchronize(dev)
    fwd_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)) / steps
    bwd_ms = sum(ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(steps)) / steps
    # the three attention kernels alone (event pairs around them)
    ops.kernel_timer_enable(True)
    for _ in range(steps):
        fwd()
        bwd()
    kms, nk = ops.kernel_timer_read()
    ops.kernel_timer_enable(False)
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out in the QAT loop")
    flops, pairs = qat_flops(w, inp["lengths"])
    step_ms = fwd_ms + bwd_ms
    attn_ms = kms / steps
    p16, src = peaks["bf16_tflops_sustained"], peak_src
    achieved = flops / (attn_ms * 1e-3) / 1e12
    line = {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "d": w.d,
            "causal": w.causal, "blk": w.blk, "dtype": "bf16",
            "step": "forward (quantise, O, O', lse) + backward (dQ, dK, dV) reusing the "
                    "forward's fake-quantised images",
            "value": flops / (step_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": step_ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "attention_kernels_ms": attn_ms, "algorithmic_flops": flops,
            "roofline": {"bound": "tensor", "kernel": "qat_fwd + qat_bwd_kv + qat_bwd_q",
                         "achieved": achieved, "peak": p16, "unit": "TFLOP/s",
                         "frac": achieved / p16, "traffic": qat_traffic(w),
                         "peak_note": f"{src} bf16 sustained (the kernels run 16-bit MMAs)",
                         "executed_mma_flops": 14 * 2 * pairs * w.d,
                         "note": "7 algorithmic products; the kernels execute 14 (S recomputed "
                                 "in each pass, dS and the P of O' as two 16-bit parts)"},
            "kernels_per_step": QAT_KERNELS_PER_STEP, "steps": steps}
    if not args.no_cpu_baseline:
        # the oracle on a causal prefix of kv head 0 with its query heads: a
        # complete smaller problem of the same shape per head
        import oracle
        cores = os.cpu_count() or 1
        L = 1024
        grp = w.H // w.Hkv
        host = synth.make_qat_inputs(w)
        sl = {n: synth.as_u16(host[n][:L, :grp].contiguous()) for n in ("q", "dout")}
        sl.update({n: synth.as_u16(host[n][:L, :1].contiguous()) for n in ("k", "v")})
        t0 = time.perf_counter()
        oracle.attn_qat_bwd(sl["q"], sl["k"], sl["v"], sl["dout"], synth.dtype_code(w.dtype),
                            np.array([0, L], np.int32), w.blk, w.causal, nthreads=cores)
        dt = time.perf_counter() - t0
        fl = 7 * 2 * (L * (L + 1) // 2) * grp * w.d
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle", "seconds": dt,
                                "sample": f"first {L} tokens of kv head 0 with its {grp} query "
                                          f"heads (a complete causal problem)"}
    del q, k, v, dout, ws, out, out_hp, lse
    torch.cuda.empty_cache()
    return line


def qat_only(args):
    """A few Attn-QAT steps (profiling aid)."""
    from bit_quantization_b200 import ops
    dev = torch.device("cuda", 0)
    w = synth.C_QAT4K
    inp, q, k, v, dout, cu, ws = qat_setup(ops, dev, w)
    times = []
    for _ in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        out, out_hp, lse = ops.thrift_qat_fwd(q, k, v, cu, w.N, blk=w.blk, causal=w.causal,
                                              workspace=ws)
        ops.thrift_qat_bwd(q, k, v, dout, out_hp, lse, cu, w.N, blk=w.blk, causal=w.causal,
                           reuse_images=True, workspace=ws)
        e1.record()
        torch.cuda.synchronize(dev)
        times.append(e0.elapsed_time(e1))
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out")
    flops, _ = qat_flops(w, inp["lengths"])
    best = min(times[args.warmup:])
    print(json.dumps({"mode": "qat", "workload": w.name, "ms_min": best,
                      "tflops": flops / (best * 1e-3) / 1e12}))
    return 0


def variant_kernel_ms(ops, q, k, v, w, out, lse, ws, frac, sink=0, recent=0, steps=20,
                      smooth=False):
    """Average attention-kernel time of the bench workload run with another
    selection or option (CUDA events around each attention launch)."""
    def step():
        ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=frac,
                            use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                            out=out, lse=lse, workspace=ws, sink_blocks=sink, recent_blocks=recent,
                            smooth_k=smooth)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ops.kernel_timer_enable(True)
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    ops.kernel_timer_enable(False)
    kms, n = ops.kernel_timer_read()
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out (selection variant)")
    return kms / max(n, 1)


def sink_line(ops, q, k, v, w, inp, out, lse, ws, p16, sink=1, recent=1):
    """ScaleSearchAttention's sink-aware variant of the bench workload: the
    first and the newest key block of every query block on the FP16 path on
    top of the top-k pairs; the attention kernel's rate against the FP4 /
    FP16 roofline of its own pair split."""
    mask = ops.block_mean_topk(q, k, w.blk, w.causal, w.topk_frac, sink_blocks=sink,
                               recent_blocks=recent).cpu().numpy()
    f4, f16 = pair_flops(mask, w, inp["lengths"])
    k_ms = variant_kernel_ms(ops, q, k, v, w, out, lse, ws, w.topk_frac, sink, recent)
    t_ideal = f4 / (4.0 * p16 * 1e12) + f16 / (p16 * 1e12)
    achieved = (f4 + f16) / (k_ms * 1e-3) / 1e12
    return {"sink_blocks": sink, "recent_blocks": recent, "topk_frac": w.topk_frac,
            "kernel": "attn_fwd_kernel", "kernel_ms": k_ms, "achieved": achieved,
            "unit": "TFLOP/s", "fp16_share": f16 / (f4 + f16),
            "frac": (t_ideal / (k_ms * 1e-3))}


def smoothing_line(ops, q, k, v, w, out, lse, ws, steps=20, nrows=64):
    """K smoothing on the bench workload: the attention kernel's and the whole
    step's time with it, and the error of both variants against fp64
    attention (torch, on the GPU) on a sample of output rows."""
    dev = q.device
    k_ms = variant_kernel_ms(ops, q, k, v, w, out, lse, ws, w.topk_frac, smooth=True)

    def step_ms(smooth):
        for _ in range(3):
            ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=w.topk_frac,
                                out=out, lse=lse, workspace=ws, smooth_k=smooth)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=w.topk_frac,
                                out=out, lse=lse, workspace=ws, smooth_k=smooth)
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    gen = torch.Generator().manual_seed(11)
    rows = torch.randint(0, w.N, (nrows,), generator=gen).tolist()
    heads = torch.randint(0, w.H, (nrows,), generator=gen).tolist()
    g = w.H // w.Hkv
    err = {}
    for smooth in (False, True):
        ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=w.topk_frac, out=out,
                            lse=lse, workspace=ws, smooth_k=smooth)
        torch.cuda.synchronize(dev)
        se = 0.0
        for t, h in zip(rows, heads):
            qr = q[0, t, h].double()
            kk = k[0, : (t + 1 if w.causal else w.N), h // g].double()
            vv = v[0, : kk.shape[0], h // g].double()
            p = torch.softmax(kk @ qr / (w.d ** 0.5), dim=0)
            se += float(((out[0, t, h].double() - p @ vv) ** 2).sum())
        err["on" if smooth else "off"] = (se / (nrows * w.d)) ** 0.5
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out (smoothing)")
    return {"kernel": "attn_fwd_kernel", "kernel_ms": k_ms, "step_ms": step_ms(True),
            "step_ms_without": step_ms(False),
            "rms_err_vs_fp64": err, "sample": f"{nrows} (token, head) rows of batch entry 0",
            "reference": "torch fp64 softmax(q K^T / sqrt(d)) V of the 16-bit inputs"}


def nvfp4_only_line(ops, q, k, v, w, out, lse, ws, flops, p4, steps=20):
    """The attention kernel with no FP16 pairs (topk_frac = 0): every score
    on the NVFP4 path, against the FP4 tensor peak alone."""
    def step():
        ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=0.0,
                            use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                            out=out, lse=lse, workspace=ws)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ops.kernel_timer_enable(True)
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    ops.kernel_timer_enable(False)
    kms, n = ops.kernel_timer_read()
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out (topk_frac = 0)")
    k_ms = kms / max(n, 1)
    achieved = flops / (k_ms * 1e-3) / 1e12
    return {"topk_frac": 0.0, "kernel": "attn_fwd_kernel", "kernel_ms": k_ms,
            "achieved": achieved, "peak": p4, "unit": "TFLOP/s", "frac": achieved / p4}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="b2h32n8192", choices=sorted(WORKLOADS))
    ap.add_argument("--ref-units", type=int, default=24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quantizer", action="store_true")
    ap.add_argument("--mode", default="attention",
                    choices=["attention", "quantizer", "decode", "qat"],
                    help="quantizer / decode: only a few plain calls of that path (profiling aid)")
    ap.add_argument("--decode-context", type=int, default=None,
                    help="cached tokens per sequence in --mode decode (default: the workload's)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-qat", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mode == "quantizer":
        return quantizer_only(args)
    if args.mode == "decode":
        return decode_only(args)
    if args.mode == "qat":
        return qat_only(args)

    from bit_quantization_b200 import ops
    world, rank, local = dist.setup("nccl")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()

    inp = synth.make_attn_inputs(w, seed=dist.rank_seed(w.seed, rank))
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(ops.thrift_attn_workspace_size(w.B, w.H, w.Hkv, w.N, w.d, w.blk),
                     dtype=torch.uint8, device=dev)

    def step(qq, kk, vv):
        ops.thrift_attn_fwd(qq, kk, vv, blk=w.blk, causal=w.causal, topk_frac=w.topk_frac,
                            use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                            out=out, lse=lse, workspace=ws)

    # FLOP split from the selection this input produces
    mask = ops.block_mean_topk(q, k, w.blk, w.causal, w.topk_frac).cpu().numpy()
    f4, f16 = pair_flops(mask, w, inp["lengths"])
    flops = f4 + f16

    for _ in range(args.warmup):
        step(q, k, v)
    torch.cuda.synchronize(dev)
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out during warm-up")

    sampler = ClockSampler(dev)
    dist.barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    ops.kernel_timer_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step(q, k, v)
    e1.record()
    torch.cuda.synchronize(dev)
    ops.kernel_timer_enable(False)
    clocks = sampler.stop()
    dist.barrier(world)
    ms_total = e0.elapsed_time(e1)
    kms, klaunches = ops.kernel_timer_read()
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out during the timed region")
    ms_total, k_ms = dist.max_over_ranks([ms_total, kms / max(klaunches, 1)], world)
    ms_step = ms_total / args.steps
    job_flops = dist.sum_over_ranks([flops], world)[0]
    value = dist.whole_job_rate(job_flops, ms_step) / 1e12

    # End to end through the public API with host buffers: every step copies
    # its Q, K, V from pinned host memory and reads its output and LSE back.
    # Steps are pipelined the way a serving loop streams batches: step s+1's
    # inputs go up on a copy stream and step s-1's results come down on
    # another while step s computes (two device buffer sets).
    qh, kh, vh = (inp[n].pin_memory() for n in ("q", "k", "v"))
    outh = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    lseh = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    qd = [torch.empty_like(q) for _ in range(2)]
    kd = [torch.empty_like(k) for _ in range(2)]
    vd = [torch.empty_like(v) for _ in range(2)]
    od = [torch.empty_like(out) for _ in range(2)]
    ld = [torch.empty_like(lse) for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(4, min(args.steps, 30))

    def e2e_run(nsteps):
        for st in range(nsteps):
            b = st % 2
            with torch.cuda.stream(s_in):
                if st >= 2:
                    s_in.wait_event(ev_comp[b])  # step st-2 has consumed buffer b
                qd[b].copy_(qh, non_blocking=True)
                kd[b].copy_(kh, non_blocking=True)
                vd[b].copy_(vh, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[b])
                if st >= 2:
                    s_comp.wait_event(ev_out[b])  # step st-2's results have left buffer b
                ops.thrift_attn_fwd(qd[b], kd[b], vd[b], blk=w.blk, causal=w.causal,
                                    topk_frac=w.topk_frac, use_scalesearch=w.use_scalesearch,
                                    use_hadamard=w.use_hadamard, out=od[b], lse=ld[b],
                                    workspace=ws)
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                outh[b].copy_(od[b], non_blocking=True)
                lseh[b].copy_(ld[b], non_blocking=True)
                ev_out[b].record(s_out)

    e2e_run(2)
    torch.cuda.synchronize(dev)
    dist.barrier(world)
    torch.cuda.synchronize(dev)
    e0.record()
    e2e_run(e2e_steps)
    for sx in (s_in, s_comp, s_out):
        torch.cuda.current_stream(dev).wait_stream(sx)
    e1.record()
    torch.cuda.synchronize(dev)
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError("device wait timed out in the end-to-end loop")
    e2e_ms = dist.max_over_ranks([e0.elapsed_time(e1)], world)[0] / e2e_steps
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
    d2h = outh[0].numel() * outh[0].element_size() + lseh[0].numel() * lseh[0].element_size()

    # roofline of the attention kernel (dominant): tensor-bound contraction;
    # t_ideal = F4/P4 + F16/P16 with P16 the measured bf16 GEMM rate and
    # P4 = 4 x P16 (nominal dense FP4 : BF16 ratio).
    p16 = peaks["bf16_tflops_sustained"]
    p4 = 4.0 * p16
    t_ideal_ms = (f4 / (p4 * 1e12) + f16 / (p16 * 1e12)) * 1e3
    achieved = flops / (k_ms * 1e-3) / 1e12
    peak_eff = flops / (t_ideal_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attn_fwd_kernel", "achieved": achieved,
                "peak": peak_eff, "unit": "TFLOP/s", "frac": achieved / peak_eff,
                "traffic": attn_traffic(w),
                "peak_note": (f"{peak_src} bf16 sustained {p16} TF/s x4 for the FP4 share, x1 for "
                              f"the FP16 share ({100 * f16 / flops:.1f}% of flops)"),
                "kernel_ms": k_ms, "fp4_flops": f4, "fp16_flops": f16}

    # ALU roofline of the same kernel: the MUFU operations per score element
    # (XU_OPS_PER_ELEMENT) against the MUFU lanes of the SMs.
    sm_mhz = clocks.get("sm_mhz") or 1965.0
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    elems = flops / (4.0 * w.d)
    alu_peak = XU_OPS_PER_CLK_PER_SM * n_sm * sm_mhz * 1e6 / XU_OPS_PER_ELEMENT / 1e9
    alu_achieved = elems / (k_ms * 1e-3) / 1e9
    alu_roofline = {"bound": "alu", "kernel": "attn_fwd_kernel", "achieved": alu_achieved,
                    "peak": alu_peak, "unit": "Gelem/s", "frac": alu_achieved / alu_peak,
                    "peak_note": (f"{XU_OPS_PER_CLK_PER_SM} MUFU lanes per SM x {n_sm} SMs x "
                                  f"{sm_mhz:.0f} MHz / {XU_OPS_PER_ELEMENT} ops per score element"),
                    "tflops_equivalent_peak": alu_peak * 1e9 * 4 * w.d / 1e12}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4+bf16",
            "data": "synthetic", "config": config_of(w), "roofline": roofline,
            "alu_roofline": alu_roofline,
            "e2e": {"value": dist.whole_job_rate(job_flops, e2e_ms) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "pipelining": "inputs of step s+1 and results of step s-1 copied while "
                                  "step s computes (two buffer sets, three streams)"},
            "gpu_launches": KERNELS_PER_STEP * args.steps, "clocks": clocks}
    if rank == 0 and world == 1:
        line["nvfp4_only"] = nvfp4_only_line(ops, q, k, v, w, out, lse, ws, flops, p4)
        line["sink_aware"] = sink_line(ops, q, k, v, w, inp, out, lse, ws, p16)
        if not w.use_hadamard:
            line["k_smoothing"] = smoothing_line(ops, q, k, v, w, out, lse, ws)
    if rank == 0 and world == 1 and not args.no_quantizer:
        line["quantizer"] = quantizer_line(dev, peaks)
    if rank == 0 and world == 1 and not args.no_decode:
        del qd, kd, vd, od, ld
        torch.cuda.empty_cache()
        line["decode"] = decode_line(ops, dev, peaks)
    if rank == 0 and world == 1 and not args.no_qat:
        line["qat"] = qat_line(ops, dev, peaks, peak_src, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        dt, fl, desc = oracle_sample(w, args.ref_units, cores, inp)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores,
                                "kind": "oracle", "sample": desc, "seconds": dt}
    dist.teardown(world)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
