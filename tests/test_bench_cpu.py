"""Host-side arithmetic of bench.py: the FLOP counts its throughput numbers
divide by, and the guards that drop recorded ncu traffic once a kernel
source changes.  No device needed."""
import dataclasses
import importlib.util
import os

import numpy as np

from bit_quantization_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_pair_flops_counts_visible_score_elements():
    b = _bench()
    w = dataclasses.replace(synth.TINY, N=256, H=2, blk=64, causal=True)
    nb = 4
    mask = np.zeros((1, w.H, nb, nb), np.uint8)
    mask[0, 1, 3, 0] = 1  # one FP16 pair of head 1: a full 64 x 64 block below the diagonal
    f4, f16 = b.pair_flops(mask, w, [256])
    visible = 256 * 257 // 2  # causal score elements per head
    assert f4 + f16 == 4 * w.d * visible * w.H
    assert f16 == 4 * w.d * 64 * 64
    wn = dataclasses.replace(w, causal=False)
    f4n, f16n = b.pair_flops(mask, wn, [256])
    assert f4n + f16n == 4 * w.d * 256 * 256 * w.H


def test_qat_flops_are_seven_products_per_visible_pair():
    b = _bench()
    w = dataclasses.replace(synth.C_QAT4K, H=4, Hkv=2, N=100)
    flops, pairs = b.qat_flops(w, [100, 37])
    assert pairs == (100 * 101 // 2 + 37 * 38 // 2) * 4
    assert flops == 7 * 2 * pairs * w.d
    wn = dataclasses.replace(w, causal=False)
    _, pn = b.qat_flops(wn, [100, 37])
    assert pn == (100 * 100 + 37 * 37) * 4


def test_recorded_traffic_only_for_its_workload():
    b = _bench()
    assert b.qat_traffic(dataclasses.replace(synth.C_QAT4K, name="other")) is None
    assert b.attn_traffic(dataclasses.replace(synth.C_B2H32N8K, name="other")) is None
    t = b.qat_traffic(synth.C_QAT4K)
    # either the source is the one the counters were taken on, or nothing
    assert t is None or t == b.QAT_TRAFFIC["bytes"]


def test_tensor_roofline_splits_the_ideal_time_by_precision():
    b = _bench()
    peaks = {"bf16_tflops": 1000.0}
    # pure NVFP4: the ideal is F / (4 x the bf16 rate)
    r = b.tensor_roofline(4e12, 0.0, 2.0, peaks, "measured")
    assert abs(r["achieved"] - 2000.0) < 1e-9
    assert abs(r["peak"] - 4000.0) < 1e-9
    assert abs(r["frac"] - 0.5) < 1e-12
    # mixed: t_ideal = 3e12 / 4e15 + 1e12 / 1e15 = 1.75 ms; the kernel took 3.5 ms
    r = b.tensor_roofline(3e12, 1e12, 3.5, peaks, "measured")
    assert abs(r["frac"] - 0.5) < 1e-12
    assert abs(r["peak"] - 4e12 / 1.75e-3 / 1e12) < 1e-9
    # the fraction against the nominal dense peaks uses their own ideal time
    t_nom = 3e12 / (b.NOMINAL_FP4_TFLOPS * 1e12) + 1e12 / (b.NOMINAL_BF16_TFLOPS * 1e12)
    assert abs(r["frac_of_nominal"] - t_nom / 3.5e-3) < 1e-12


def test_alu_roofline_counts_score_elements():
    b = _bench()
    d, n_sm, mhz = 128, 148, 2000.0
    flops = 4 * d * 1e9  # 1e9 score elements
    r = b.alu_roofline(flops, d, 1.0, mhz, n_sm)
    assert abs(r["achieved"] - 1000.0) < 1e-9  # Gelem/s
    peak = b.XU_OPS_PER_CLK_PER_SM * n_sm * mhz * 1e6 / b.XU_OPS_PER_ELEMENT / 1e9
    assert abs(r["peak"] - peak) < 1e-9
    assert abs(r["tflops_equivalent_peak"] - peak * 1e9 * 4 * d / 1e12) < 1e-6
