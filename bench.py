#!/usr/bin/env python
"""Benchmark of the NVFP4 / selective-FP16 attention forward on B200.

One step = one attention call over one batch of the workload: tensor absmax,
Q/K/V NVFP4 quantisation (Hadamard and ScaleSearch when the workload asks),
block-mean top-k selection and the mixed NVFP4/FP16 attention kernel.
Prints one JSON line (rank 0).

Headline workload (default): the largest single-GPU configuration, causal
GQA B=1, H=32, Hkv=8, N=32768, d=128, bf16, 128x128 blocks, 128-point
Hadamard on Q/K, ScaleSearch, 5% FP16 pairs, K with per-channel offsets
N(0, 3).  Its inputs (268 + 2 x 67 MB) exceed L2, so no flush is needed
between steps.

The line also carries one object per other attention configuration ("configs":
B2 H32 N8192 non-causal top 10%, and the varlen batch of 16 sequences at top
0/5/25%), each with its own kernel roofline, oracle time and error against
unquantised fp64 attention; the quantiser workload ("quantizer"); one decode
step over the double cache ("decode"); and one Attn-QAT training step ("qat").

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
    "gqa32k": synth.C_GQA32K,
    "b2h32n8192": synth.C_B2H32N8K,
    "varlen": synth.C_VARLEN,
    "tiny": synth.TINY,
}
# The other attention configurations reported beside the headline, each as
# its own object: (key, workload).
SECONDARY = [
    ("b2h32n8192_top10", synth.C_B2H32N8K),
    ("varlen_top0", dataclasses.replace(synth.C_VARLEN, topk_frac=0.0)),
    ("varlen_top5", dataclasses.replace(synth.C_VARLEN, topk_frac=0.05)),
    ("varlen_top25", dataclasses.replace(synth.C_VARLEN, topk_frac=0.25)),
]

METRIC = "NVFP4 attention fwd TFLOPS (whole step: quantise + select + attention)"
UNIT = "TFLOP/s"
# 3 absmax, 2 Q/K images (with the block means), 1 V image, 1 scores, 1 top-k,
# 1 attention
KERNELS_PER_STEP = 9
# Nominal dense peaks of one B200 (context beside the measured ones)
NOMINAL_FP4_TFLOPS = 9000.0
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _src_sha(name):
    import hashlib
    with open(os.path.join(ROOT, "bit_quantization_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# DRAM traffic of one attention launch measured by ncu (read + write bytes)
# per workload, for the attention source with this hash; reported only while
# the source is unchanged since the capture.
ATTN_TRAFFIC = {"src_sha16": "abe4ba02cd17350b",
                "bytes": {"b2h32n8192d128_bf16_noncausal_top10": 395558144 + 121920256,
                          "b1h32hkv8n32768d128_bf16_causal_had_ss_top5": 499836672}}


def attn_traffic(w):
    if _src_sha("attn.cuh") == ATTN_TRAFFIC["src_sha16"]:
        return ATTN_TRAFFIC["bytes"].get(w.name)
    return None


# DRAM traffic per step of the three Attn-QAT attention kernels (forward,
# key-tile and query-tile backward) from the ncu launch list of the QAT source
# with this hash (per-launch means over five steps); reported only while the
# source is unchanged.
QAT_TRAFFIC = {"src_sha16": "494a53898754d554", "workload": "qat_b1h32hkv8n4096d128_bf16_causal",
               "bytes": int((96.3 + 90.2 + 107.3) * 1e6)}


def qat_traffic(w):
    if _src_sha("qat.cuh") == QAT_TRAFFIC["src_sha16"] and w.name == QAT_TRAFFIC["workload"]:
        return QAT_TRAFFIC["bytes"]
    return None


XU_OPS_PER_CLK_PER_SM = 16   # MUFU lanes per SM (4 per sub-partition)
# MUFU operations per score element: one exp2, plus one exp2 and one log2 per
# 16-key block for the block scale (the E2M1 / 16-bit converts do not use
# this pipe: an instruction-class count of each convert shows none there)
XU_OPS_PER_ELEMENT = 1.125
# Warp instructions one sub-partition issues per clock (4 per SM)
ISSUE_PER_CLK_PER_SM = 4


def pair_flops(mask, w, lengths):
    """Algorithmic FLOPs (4*d per unmasked score element) split by path.
    mask [nseq, H, nB, nB] (1 = FP16 pair); sequence b uses its first
    ceil(L_b / blk) block rows and columns."""
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


def tensor_roofline(f4, f16, k_ms, peaks, peak_src):
    """Roofline of the attention kernel: a tensor-bound contraction with
    t_ideal = F4 / P4 + F16 / P16.  P16 is the measured bf16 GEMM burst rate
    (the kernel is timed over tens of milliseconds, not a seconds-long
    power-capped loop) and P4 = 4 x P16 (the nominal dense FP4 : BF16 ratio).
    The same fraction against the nominal dense peaks is given beside it."""
    p16 = peaks["bf16_tflops"]
    p4 = 4.0 * p16
    flops = f4 + f16
    t_ideal = f4 / (p4 * 1e12) + f16 / (p16 * 1e12)
    t_nom = f4 / (NOMINAL_FP4_TFLOPS * 1e12) + f16 / (NOMINAL_BF16_TFLOPS * 1e12)
    achieved = flops / (k_ms * 1e-3) / 1e12
    peak_eff = flops / t_ideal / 1e12
    return {"bound": "tensor", "kernel": "attn_fwd_kernel", "achieved": achieved,
            "peak": peak_eff, "unit": "TFLOP/s", "frac": achieved / peak_eff,
            "peak_note": (f"{peak_src} bf16 burst {p16} TF/s x4 for the FP4 share, x1 for the "
                          f"FP16 share ({100 * f16 / max(flops, 1):.1f}% of flops)"),
            "frac_of_nominal": t_nom / (k_ms * 1e-3),
            "nominal_note": f"against nominal dense {NOMINAL_FP4_TFLOPS:.0f} TF/s FP4 and "
                            f"{NOMINAL_BF16_TFLOPS:.0f} TF/s BF16",
            "kernel_ms": k_ms, "fp4_flops": f4, "fp16_flops": f16}


def alu_roofline(flops, d, k_ms, sm_mhz, n_sm):
    """ALU roofline of the attention kernel: the MUFU operations per score
    element (XU_OPS_PER_ELEMENT) against the MUFU lanes of the SMs."""
    elems = flops / (4.0 * d)
    peak = XU_OPS_PER_CLK_PER_SM * n_sm * sm_mhz * 1e6 / XU_OPS_PER_ELEMENT / 1e9
    achieved = elems / (k_ms * 1e-3) / 1e9
    return {"bound": "alu", "kernel": "attn_fwd_kernel", "achieved": achieved, "peak": peak,
            "unit": "Gelem/s", "frac": achieved / peak,
            "peak_note": (f"{XU_OPS_PER_CLK_PER_SM} MUFU lanes per SM x {n_sm} SMs x "
                          f"{sm_mhz:.0f} MHz / {XU_OPS_PER_ELEMENT} ops per score element"),
            "tflops_equivalent_peak": peak * 1e9 * 4 * d / 1e12}


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
    """The CPU oracle on a bounded sample of the workload: one head of the
    first sequence (full length), `nunits` evenly spread query blocks.
    Returns (seconds, algorithmic flops of the sampled rows, description)."""
    import oracle
    if inp is None:
        inp = synth.make_attn_inputs(w)
    d, blk = w.d, w.blk
    N = inp["lengths"][0]
    if w.varlen is None:
        q, k, v = (inp[n][0, :, 0:1].contiguous() for n in ("q", "k", "v"))
    else:
        q, k, v = (inp[n][:N, 0:1].contiguous() for n in ("q", "k", "v"))
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
        fl += 4.0 * d * float(cnt)
    nheads = w.B * w.H if w.varlen is None else len(inp["lengths"]) * w.H
    desc = (f"1 of {nheads} (sequence, head) problems (sequence 0, head 0, full length {N}), "
            f"{len(blocks)} of {nb} query blocks; includes that head's quantisation and "
            f"selection")
    return dt, fl, desc


def cpu_baseline(w, inp, budget_s=10.0, max_units=64):
    """The oracle timed on the host cores on a sample sized to about
    `budget_s` seconds, its rate in the line's unit."""
    cores = os.cpu_count() or 1
    dt0, fl0, _ = oracle_sample(w, 2, cores, inp)
    units = int(max(2, min(max_units, 2 * budget_s / max(dt0, 1e-3))))
    dt, fl, desc = oracle_sample(w, units, cores, inp)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": desc, "seconds": dt}


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
            "data": "synthetic", "config": config_of(w, inp["lengths"]),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, lengths=None):
    c = {"workload": w.name, "B": w.B, "H": w.H, "Hkv": w.Hkv, "N": w.N, "d": w.d,
         "dtype": str(w.dtype).replace("torch.", ""), "causal": w.causal, "blk": w.blk,
         "topk_frac": w.topk_frac, "scalesearch": w.use_scalesearch,
         "hadamard": w.use_hadamard, "k_offset_std": w.k_offset_std,
         "l2": "inputs larger than L2 (no flush)", "parallelism": "independent problems per GPU"}
    if w.varlen is not None:
        c.update({"nseq": len(lengths), "lengths": list(lengths), "total_tokens": int(sum(lengths))})
        c["B"] = len(lengths)
    return c


# Issue slots per element of the ScaleSearch-on quantiser, from a one-launch
# ncu capture of quant_rows_kernel<fp16, no rotation, ScaleSearch> on the
# quantiser workload: 21.09 M warp instructions for 524 288 16-element blocks
# (one block per thread) = 1287 per block = 80.4 per element.  A count from the
# source (9 candidates x ~110 instructions + ~86) gives 67; the measured count
# is the denominator.
QUANT_SS_ISSUE_PER_ELEM = 80.4
QUANT_SS_ISSUE_NOTE = ("issue slots per element measured by ncu (smsp__inst_executed.sum of "
                       "one launch x 32 lanes / elements; ~1290 per 16-block)")


def quantizer_line(dev, peaks, with_oracle=True):
    """Quantiser-only workload (65536 x 128 fp16 with 4 outlier channels):
    GB/s of algorithmic bytes (2 B read + 0.5625 B written per element).
    Twelve rotating input copies (> L2); the calls are captured in one CUDA
    graph so host-side launch gaps do not enter the timing.  The oracle
    quantises the whole tensor on the host cores beside it."""
    from bit_quantization_b200 import ops
    x0 = synth.make_quant_input(synth.QUANT).to(dev)
    xs = [x0.clone() for _ in range(12)]
    rows, cols = x0.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=dev)
    ws = torch.empty(ops.lib().nvfp4_quantize_workspace_size(), dtype=torch.uint8, device=dev)
    res = {}
    elems = rows * cols
    algo = elems * (2 + 0.5 + 0.0625)
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
                    "frac_of_nominal_hbm": gbs / NOMINAL_HBM_GBS}
        if ss:
            n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
            clk = peaks.get("sm_max_mhz", 1965.0)
            peak_elem = ISSUE_PER_CLK_PER_SM * 32 * n_sm * clk * 1e6 / QUANT_SS_ISSUE_PER_ELEM
            ach_elem = elems / (ms * 1e-3)
            res[key]["alu_roofline"] = {
                "bound": "alu", "achieved": ach_elem / 1e9, "peak": peak_elem / 1e9,
                "unit": "Gelem/s", "frac": ach_elem / peak_elem,
                "peak_note": f"{ISSUE_PER_CLK_PER_SM} warp instructions per clock per SM x 32 "
                             f"lanes x {n_sm} SMs x {clk:.0f} MHz / {QUANT_SS_ISSUE_PER_ELEM} "
                             f"({QUANT_SS_ISSUE_NOTE})",
                "gbs_equivalent_peak": peak_elem * 2.5625 / 1e9}
        del g
    res["workload"] = synth.QUANT.name
    res["algorithmic_bytes"] = algo
    res["kernels_per_call"] = {"scale_given": 1, "scale_computed": 2}
    res["timing"] = "CUDA graph of 120 calls, 12 rotating inputs (201 MB > L2)"
    if with_oracle:
        import oracle
        cores = os.cpu_count() or 1
        xh = synth.as_u16(synth.make_quant_input(synth.QUANT))
        ob = {}
        for ss in (False, True):
            t0 = time.perf_counter()
            oracle.nvfp4_quantize(xh, synth.dtype_code(synth.QUANT.dtype), use_ss=ss)
            dt = time.perf_counter() - t0
            ob["scalesearch_on" if ss else "scalesearch_off"] = {
                "seconds": dt, "gbs": algo / dt / 1e9, "unit": "GB/s"}
        res["cpu_baseline"] = {"kind": "oracle", "cores": 1, "host_cores": cores,
                               "sample": "the whole 65536 x 128 tensor (tensor absmax, block "
                                         "scales, codes), one thread",
                               "value": ob["scalesearch_off"]["gbs"], "unit": "GB/s", **ob}
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
    ws = torch.empty(ops.qat_workspace_size(q.shape[0], w.H, w.Hkv, w.d, cu.numel() - 1),
                     dtype=torch.uint8, device=dev)
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
    p16, src = peaks["bf16_tflops"], peak_src
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
                         "peak_note": f"{src} bf16 burst (the kernels run 16-bit MMAs; the "
                                      f"timed region is tens of milliseconds)",
                         "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                         "executed_mma_flops": 12 * 2 * pairs * w.d,
                         "note": "7 algorithmic products; the kernels execute 12 (each "
                                 "gradient kernel computes S and dP again; the dS of dQ and the "
                                 "P of O' enter as two 16-bit parts)"},
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


class AttnCase:
    """One attention workload resident on the device: inputs, outputs,
    workspace and the call one step makes (the packed entry point for a
    varlen batch)."""

    def __init__(self, ops, dev, w, seed=None):
        self.ops, self.dev, self.w = ops, dev, w
        self.inp = synth.make_attn_inputs(w, seed=seed)
        self.lengths = self.inp["lengths"]
        self.q, self.k, self.v = (self.inp[n].to(dev) for n in ("q", "k", "v"))
        self.varlen = w.varlen is not None
        self.out = torch.empty_like(self.q)
        if self.varlen:
            self.nseq, self.maxlen = len(self.lengths), max(self.lengths)
            total = self.q.shape[0]
            self.cu = self.inp["cu_seqlens"].to(dev)
            self.lse = torch.empty((w.H, total), dtype=torch.float32, device=dev)
            need = ops.thrift_attn_varlen_workspace_size(self.nseq, total, self.maxlen, w.H, w.Hkv,
                                                         w.d, w.blk)
        else:
            self.nseq, self.maxlen = w.B, w.N
            self.cu = None
            self.lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
            need = ops.thrift_attn_workspace_size(w.B, w.H, w.Hkv, w.N, w.d, w.blk)
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def run(self, q=None, k=None, v=None, out=None, lse=None, frac=None, sink=0, recent=0,
            smooth=False):
        w, ops = self.w, self.ops
        q = self.q if q is None else q
        k = self.k if k is None else k
        v = self.v if v is None else v
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        frac = w.topk_frac if frac is None else frac
        if self.varlen:
            ops.thrift_attn_fwd_varlen(q, k, v, self.cu, self.maxlen, blk=w.blk, causal=w.causal,
                                       topk_frac=frac, use_scalesearch=w.use_scalesearch,
                                       use_hadamard=w.use_hadamard, out=out, lse=lse,
                                       workspace=self.ws, sink_blocks=sink, recent_blocks=recent,
                                       smooth_k=smooth)
        else:
            ops.thrift_attn_fwd(q, k, v, blk=w.blk, causal=w.causal, topk_frac=frac,
                                use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                                out=out, lse=lse, workspace=self.ws, sink_blocks=sink,
                                recent_blocks=recent, smooth_k=smooth)

    def run_sharded(self, world, q=None, k=None, v=None, out=None, lse=None):
        """One step of a problem split across `world` ranks, on this rank's
        shard (its inputs): the shard's three tensor absmaxes, their maximum
        over the ranks (one all-reduce of 3 floats), then the attention under
        the agreed absmaxes.  With one rank the same calls, no all-reduce."""
        from bit_quantization_b200 import shard
        w, ops = self.w, self.ops
        q = self.q if q is None else q
        k = self.k if k is None else k
        v = self.v if v is None else v
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        if not hasattr(self, "amax"):
            self.amax = torch.empty(3, dtype=torch.float32, device=self.dev)
        ops.thrift_attn_absmax(q, k, v, self.cu, self.maxlen, blk=w.blk,
                               use_hadamard=w.use_hadamard, amax=self.amax, workspace=self.ws)
        shard.agree_absmax(self.amax, world)
        ops.thrift_attn_fwd_absmax(q, k, v, self.amax, self.cu, self.maxlen, blk=w.blk,
                                   causal=w.causal, topk_frac=w.topk_frac,
                                   use_scalesearch=w.use_scalesearch, use_hadamard=w.use_hadamard,
                                   out=out, lse=lse, workspace=self.ws)

    def mask(self):
        """The selection [nseq, H, nB, nB] the last call left in the workspace."""
        w = self.w
        nB = (self.maxlen + w.blk - 1) // w.blk
        off = self.ops.thrift_attn_workspace_mask_offset(self.nseq, self.maxlen, w.H, w.Hkv,
                                                         w.d, w.blk)
        n = self.nseq * w.H * nB * nB
        return self.ws[off:off + n].view(self.nseq, w.H, nB, nB).cpu().numpy()

    def flops(self, **kw):
        """(F4, F16) of the selection one call with these options makes."""
        self.run(**kw)
        torch.cuda.synchronize(self.dev)
        return pair_flops(self.mask(), self.w, self.lengths)

    def kernel_ms(self, steps=20, **kw):
        """Average attention-kernel time (CUDA events around each launch on
        its stream) over `steps` calls with these options."""
        ops = self.ops
        for _ in range(3):
            self.run(**kw)
        torch.cuda.synchronize(self.dev)
        ops.kernel_timer_enable(True)
        for _ in range(steps):
            self.run(**kw)
        torch.cuda.synchronize(self.dev)
        ops.kernel_timer_enable(False)
        kms, n = ops.kernel_timer_read()
        if ops.device_status(reset=True) != ops.OK:
            raise RuntimeError("device wait timed out")
        return kms / max(n, 1)

    def err_vs_fp64(self, nrows=128, seed=11):
        """Error of the last call's output against unquantised fp64 attention
        (torch, on the device) of the same 16-bit inputs, on `nrows` seeded
        (sequence, token, head) rows; a report, not a bound."""
        w = self.w
        g = w.H // w.Hkv
        gen = torch.Generator().manual_seed(seed)
        seqs = torch.randint(0, self.nseq, (nrows,), generator=gen).tolist()
        fr = torch.rand((nrows,), generator=gen).tolist()
        heads = torch.randint(0, w.H, (nrows,), generator=gen).tolist()
        se = ref2 = 0.0
        mx = 0.0
        for s, f, h in zip(seqs, fr, heads):
            L = self.lengths[s]
            t = min(L - 1, int(f * L))
            n_keys = t + 1 if w.causal else L
            if self.varlen:
                a = int(self.inp["cu_seqlens"][s])
                qr, o = self.q[a + t, h], self.out[a + t, h]
                kk, vv = self.k[a:a + n_keys, h // g], self.v[a:a + n_keys, h // g]
            else:
                qr, o = self.q[s, t, h], self.out[s, t, h]
                kk, vv = self.k[s, :n_keys, h // g], self.v[s, :n_keys, h // g]
            p = torch.softmax(kk.double() @ qr.double() / (w.d ** 0.5), dim=0)
            ref = p @ vv.double()
            dlt = o.double() - ref
            se += float((dlt ** 2).sum())
            ref2 += float((ref ** 2).sum())
            mx = max(mx, float(dlt.abs().max()))
        n = nrows * w.d
        return {"max_abs": mx, "rms": (se / n) ** 0.5, "rms_of_reference": (ref2 / n) ** 0.5,
                "rows": nrows, "sample": "seeded uniform (sequence, token, head) rows",
                "reference": "torch fp64 softmax(q K^T / sqrt(d)) V of the 16-bit inputs"}


def nvfp4_only_object(case, peaks, peak_src, steps=20):
    """The attention kernel with no FP16 pairs (topk_frac = 0): every score
    on the NVFP4 path, against the FP4 tensor peak alone."""
    f4, f16 = case.flops(frac=0.0)
    k_ms = case.kernel_ms(steps, frac=0.0)
    p4 = 4.0 * peaks["bf16_tflops"]
    achieved = (f4 + f16) / (k_ms * 1e-3) / 1e12
    return {"topk_frac": 0.0, "kernel": "attn_fwd_kernel", "kernel_ms": k_ms,
            "achieved": achieved, "peak": p4, "unit": "TFLOP/s", "frac": achieved / p4,
            "peak_note": f"{peak_src} bf16 burst x4",
            "frac_of_nominal": achieved / NOMINAL_FP4_TFLOPS}


def sink_object(case, peaks, peak_src, sink=1, recent=1):
    """ScaleSearchAttention's sink-aware variant: the first and the newest key
    block of every query block on the FP16 path on top of the top-k pairs;
    the attention kernel's rate against the FP4 / FP16 roofline of its own
    pair split."""
    f4, f16 = case.flops(sink=sink, recent=recent)
    k_ms = case.kernel_ms(sink=sink, recent=recent)
    r = tensor_roofline(f4, f16, k_ms, peaks, peak_src)
    return {"sink_blocks": sink, "recent_blocks": recent, "topk_frac": case.w.topk_frac,
            "kernel": "attn_fwd_kernel", "kernel_ms": k_ms, "achieved": r["achieved"],
            "unit": "TFLOP/s", "fp16_share": f16 / (f4 + f16), "frac": r["frac"]}


def smoothing_object(case, steps=20):
    """K smoothing: the attention kernel's and the whole step's time with it,
    and the error of both variants against fp64 attention."""
    dev = case.dev
    k_ms = case.kernel_ms(smooth=True)

    def step_ms(smooth):
        for _ in range(3):
            case.run(smooth=smooth)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            case.run(smooth=smooth)
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    err = {}
    for smooth in (False, True):
        case.run(smooth=smooth)
        torch.cuda.synchronize(dev)
        err["on" if smooth else "off"] = case.err_vs_fp64(64)["rms"]
    if case.ops.device_status(reset=True) != case.ops.OK:
        raise RuntimeError("device wait timed out (smoothing)")
    return {"kernel": "attn_fwd_kernel", "kernel_ms": k_ms, "step_ms": step_ms(True),
            "step_ms_without": step_ms(False), "rms_err_vs_fp64": err,
            "reference": "torch fp64 softmax(q K^T / sqrt(d)) V of the 16-bit inputs"}


def config_object(case, peaks, peak_src, steps, sm_mhz, n_sm, with_cpu=True,
                  with_nvfp4_only=False):
    """One attention configuration: whole-step rate, the attention kernel's
    tensor and ALU rooflines, error against fp64 attention and the oracle on
    the host cores."""
    ops, w, dev = case.ops, case.w, case.dev
    f4, f16 = case.flops()
    flops = f4 + f16
    for _ in range(3):
        case.run()
    torch.cuda.synchronize(dev)
    ops.kernel_timer_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        case.run()
    e1.record()
    torch.cuda.synchronize(dev)
    ops.kernel_timer_enable(False)
    kms, n = ops.kernel_timer_read()
    if ops.device_status(reset=True) != ops.OK:
        raise RuntimeError(f"device wait timed out ({w.name})")
    step_ms = e0.elapsed_time(e1) / steps
    k_ms = kms / max(n, 1)
    obj = {"workload": w.name, "config": config_of(w, case.lengths),
           "value": flops / (step_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": step_ms,
           "steps": steps, "kernel_ms": k_ms, "algorithmic_flops": flops,
           "roofline": tensor_roofline(f4, f16, k_ms, peaks, peak_src),
           "alu_roofline": alu_roofline(flops, w.d, k_ms, sm_mhz, n_sm),
           "err_vs_fp64": case.err_vs_fp64(), "gpu_launches": KERNELS_PER_STEP * steps}
    obj["roofline"]["traffic"] = attn_traffic(w)
    if with_nvfp4_only:
        obj["nvfp4_only"] = nvfp4_only_object(case, peaks, peak_src)
    if with_cpu:
        obj["cpu_baseline"] = cpu_baseline(w, case.inp)
    return obj


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gqa32k", choices=sorted(WORKLOADS))
    ap.add_argument("--ref-units", type=int, default=24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quantizer", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the objects of the other attention configurations")
    ap.add_argument("--mode", default="attention",
                    choices=["attention", "quantizer", "decode", "qat"],
                    help="quantizer / decode / qat: only a few plain calls of that path "
                         "(profiling aid)")
    ap.add_argument("--decode-context", type=int, default=None,
                    help="cached tokens per sequence in --mode decode (default: the workload's)")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="tokens per sequence of a fixed-length workload (profiling a smaller case)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-qat", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = WORKLOADS[args.workload]
    if args.seq_len is not None and w.varlen is None:
        w = dataclasses.replace(w, N=args.seq_len, name=f"{w.name}_n{args.seq_len}")
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
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count

    case = AttnCase(ops, dev, w, seed=dist.rank_seed(w.seed, rank))
    # FLOP split from the selection this input produces
    f4, f16 = case.flops()
    flops = f4 + f16

    # Each rank holds one shard (its own batch entries: seed + rank) of one
    # problem of world x B sequences; the step agrees the tensor absmaxes
    # across ranks by one max all-reduce of 3 floats (NCCL), so every code is
    # the one-GPU run's of that whole problem.
    for _ in range(args.warmup):
        case.run_sharded(world)
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
        case.run_sharded(world)
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
    qh, kh, vh = (case.inp[n].pin_memory() for n in ("q", "k", "v"))
    outh = [torch.empty(case.out.shape, dtype=case.out.dtype).pin_memory() for _ in range(2)]
    lseh = [torch.empty(case.lse.shape, dtype=case.lse.dtype).pin_memory() for _ in range(2)]
    qd = [torch.empty_like(case.q) for _ in range(2)]
    kd = [torch.empty_like(case.k) for _ in range(2)]
    vd = [torch.empty_like(case.v) for _ in range(2)]
    od = [torch.empty_like(case.out) for _ in range(2)]
    ld = [torch.empty_like(case.lse) for _ in range(2)]
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
                case.run_sharded(world, qd[b], kd[b], vd[b], od[b], ld[b])
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
    del qd, kd, vd, od, ld, outh, lseh
    sm_mhz = clocks.get("sm_mhz") or 1965.0

    roofline = tensor_roofline(f4, f16, k_ms, peaks, peak_src)
    roofline["traffic"] = attn_traffic(w)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4+bf16",
            "data": "synthetic", "config": dict(config_of(w, case.lengths), parallelism=(
                f"one problem of {world} x {w.B if w.varlen is None else len(case.lengths)} "
                f"sequences split by batch across {world} GPU(s); per step one max all-reduce "
                f"of the 3 tensor absmaxes")), "roofline": roofline,
            "alu_roofline": alu_roofline(flops, w.d, k_ms, sm_mhz, n_sm),
            "e2e": {"value": dist.whole_job_rate(job_flops, e2e_ms) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "pipelining": "inputs of step s+1 and results of step s-1 copied while "
                                  "step s computes (two buffer sets, three streams)"},
            "gpu_launches": KERNELS_PER_STEP * args.steps, "clocks": clocks}
    if rank == 0 and world == 1:
        case.run()
        torch.cuda.synchronize(dev)
        line["err_vs_fp64"] = case.err_vs_fp64()
        line["nvfp4_only"] = nvfp4_only_object(case, peaks, peak_src)
        line["sink_aware"] = sink_object(case, peaks, peak_src)
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, case.inp)
    del case
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_configs:
        configs = {}
        for key, cw in SECONDARY:
            if cw.name == w.name and cw.topk_frac == w.topk_frac:
                continue
            c = AttnCase(ops, dev, cw)
            configs[key] = config_object(c, peaks, peak_src, 20, sm_mhz, n_sm,
                                         with_cpu=not args.no_cpu_baseline,
                                         with_nvfp4_only=cw is synth.C_B2H32N8K)
            if cw is synth.C_B2H32N8K:
                configs[key]["k_smoothing"] = smoothing_object(c)
            del c
            torch.cuda.empty_cache()
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_quantizer:
        line["quantizer"] = quantizer_line(dev, peaks, with_oracle=not args.no_cpu_baseline)
    if rank == 0 and world == 1 and not args.no_decode:
        line["decode"] = decode_line(ops, dev, peaks)
    if rank == 0 and world == 1 and not args.no_qat:
        line["qat"] = qat_line(ops, dev, peaks, peak_src, args)
    dist.teardown(world)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
