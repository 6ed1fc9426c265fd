"""Attention parity at the full workload sizes, in the launch configuration
the bench times: the GPU computes every output; the oracle computes the
whole quantisation and selection and then a sample of query blocks (first,
last, middle and diagonal-heavy ones), compared row by row with the bar of
test_attn_gpu.py.  Also the longest sequence a call accepts (512 key tiles).
Each case also prints its error against unquantised fp64 attention on the
sampled rows (a report, not a bound).
"""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops, synth

from test_attn_gpu import MIN_COS, _compare

pytestmark = pytest.mark.gpu


def _units_for(lengths, H, blk, picks):
    units = []
    for s, h, where in picks:
        nb = (lengths[s] + blk - 1) // blk
        i = {"first": 0, "last": nb - 1, "mid": nb // 2, "q1": nb // 4}[where] if isinstance(where, str) else where
        units.append((s, h, i))
    return np.array(units, np.int32)


def _check_units(orc, got, r, cu, units, blk, dtype):
    rows = []
    for s, h, i in units:
        a = cu[s] + i * blk
        b = min(cu[s + 1], a + blk)
        rows.append((slice(a, b), h))
    g = np.concatenate([got[a, h].reshape(-1) for a, h in rows])
    w = np.concatenate([r["out64"][a, h].reshape(-1) for a, h in rows])
    t = np.concatenate([r["tol"][a, h].reshape(-1) for a, h in rows])
    err, cos = _compare(g, w, "sampled rows", dtype, t)
    assert cos >= MIN_COS
    return err


def _run(orc, w, picks, lengths=None):
    inp = synth.make_attn_inputs(w, lengths=lengths)
    q, k, v, cu_t = inp["q"], inp["k"], inp["v"], inp["cu_seqlens"]
    lengths = inp["lengths"]
    if w.varlen is None:
        out, lse = ops.thrift_attn_fwd(q.cuda(), k.cuda(), v.cuda(), blk=w.blk, causal=w.causal,
                                       topk_frac=w.topk_frac, use_scalesearch=w.use_scalesearch,
                                       use_hadamard=w.use_hadamard)
        qp, kp, vp = (synth.as_u16(t.reshape(w.B * w.N, -1, w.d)) for t in (q, k, v))
        got = out.reshape(w.B * w.N, w.H, w.d)
    else:
        out, lse = ops.thrift_attn_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_t.cuda(),
                                              max(lengths), blk=w.blk, causal=w.causal,
                                              topk_frac=w.topk_frac,
                                              use_scalesearch=w.use_scalesearch,
                                              use_hadamard=w.use_hadamard)
        qp, kp, vp = (synth.as_u16(t) for t in (q, k, v))
        got = out
    torch.cuda.synchronize()
    assert ops.device_status(reset=True) == ops.OK
    gotf = got.float().cpu().double().numpy()
    cu = cu_t.numpy()
    units = _units_for(lengths, w.H, w.blk, picks)
    r = orc.thrift_attn(qp, kp, vp, synth.dtype_code(w.dtype), cu, w.blk, w.causal, w.topk_frac,
                        use_ss=w.use_scalesearch, use_had=w.use_hadamard, units=units)
    err = _check_units(orc, gotf, r, cu, units, w.blk, w.dtype)
    # reported, not asserted: the error of the quantised result against
    # unquantised fp64 attention on the same rows
    rows = np.array([(t, h) for s, h, i in units
                     for t in range(cu[s] + i * w.blk, min(cu[s + 1], cu[s] + (i + 1) * w.blk))],
                    np.int64)
    ref, _ = orc.attn_fp64(qp, kp, vp, synth.dtype_code(w.dtype), cu, w.causal, rows=rows)
    g = gotf[rows[:, 0], rows[:, 1]].ravel()
    f = ref[rows[:, 0], rows[:, 1]].ravel()
    print(f"\n{w.name} topk {w.topk_frac}: vs unquantised fp64 attention on {len(rows)} rows: "
          f"max abs {np.abs(g - f).max():.3e}, rms {np.sqrt(np.mean((g - f) ** 2)):.3e} "
          f"(rms of the fp64 output {np.sqrt(np.mean(f ** 2)):.3e})")
    return err


def test_b2h32n8192_noncausal_top10(orc):
    w = synth.C_B2H32N8K
    _run(orc, w, [(0, 0, "first"), (0, 31, "last"), (1, 5, "mid"), (1, 17, "q1"),
                  (0, 12, 40), (1, 30, 7)])


def test_gqa32k_causal_hadamard_scalesearch_top5(orc):
    w = synth.C_GQA32K
    _run(orc, w, [(0, 0, "first"), (0, 31, "last"), (0, 9, "mid"), (0, 22, "q1"),
                  (0, 3, 200), (0, 16, 2)])


@pytest.mark.parametrize("frac", [0.0, 0.05, 0.25])
def test_varlen_batch(orc, frac):
    import dataclasses
    w = dataclasses.replace(synth.C_VARLEN, topk_frac=frac)
    _run(orc, w, [(0, 0, "first"), (3, 15, "last"), (7, 8, "mid"), (15, 2, "last"),
                  (11, 11, "q1")])


def test_longest_sequence_one_head(orc):
    # N = 65536 with 128-token blocks: 512 key tiles, the most a call accepts.
    w = synth.AttnWorkload("n65536", 1, 1, 1, 65536, 128, torch.bfloat16, True, 128, 0.05,
                           True, True, k_offset_std=3.0, seed=3)
    _run(orc, w, [(0, 0, "first"), (0, 0, "last"), (0, 0, 300)])
