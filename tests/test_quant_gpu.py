"""GPU quantiser vs the CPU oracle: codes, scales and tensor scale must be
bit-identical (ScaleSearch page: Mecanismo and Estrategia de Busqueda; the
E2M1 grid of the Attn-QAT page)."""
import numpy as np
import pytest
import torch

from bit_quantization_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _dt(dtype):
    return synth.dtype_code(dtype)


def _check_rows(orc, x, ss, had, g=None):
    codes, scales, ts = ops.nvfp4_quantize(x.cuda(), use_scalesearch=ss, use_hadamard=had,
                                           tensor_scale=None if g is None else
                                           torch.tensor([g], dtype=torch.float32, device="cuda"))
    c0, s0, g0, _ = orc.nvfp4_quantize(synth.as_u16(x), _dt(x.dtype), use_ss=ss, use_had=had, g=g)
    torch.cuda.synchronize()
    assert ops.device_status() == ops.OK
    assert ts.item() == np.float32(g0)
    sc = scales.cpu().numpy()
    cc = codes.cpu().numpy()
    assert np.array_equal(sc, s0), f"scale mismatch at {np.argwhere(sc != s0)[:5]}"
    assert np.array_equal(cc, c0), f"code mismatch at {np.argwhere(cc != c0)[:5]}"


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("ss", [False, True])
@pytest.mark.parametrize("had", [False, True])
@pytest.mark.parametrize("rows,cols", [(1000, 128), (37, 64), (1, 128)])
def test_rows_parity(orc, dtype, ss, had, rows, cols):
    x = synth.randn16((rows, cols), dtype, seed=rows + cols, scale=3.0)
    _check_rows(orc, x, ss, had)


@pytest.mark.parametrize("cols", [16, 48, 4096])
def test_rows_parity_other_widths(orc, cols):
    x = synth.randn16((97, cols), torch.bfloat16, seed=cols)
    _check_rows(orc, x, True, False)


def test_given_tensor_scale(orc):
    x = synth.randn16((256, 128), torch.float16, seed=5)
    _check_rows(orc, x, True, False, g=0.0123)


def test_zero_tensor():
    x = torch.zeros((64, 128), dtype=torch.float16, device="cuda")
    codes, scales, ts = ops.nvfp4_quantize(x, use_scalesearch=True)
    assert ts.item() == 1.0 and not codes.any() and not scales.any()


@pytest.mark.parametrize("ss", [False, True])
def test_quantizer_workload_full_size(orc, ss):
    # 65536 x 128 fp16, N(0,1) with 4 outlier channels x20.
    x = synth.make_quant_input(synth.QUANT)
    _check_rows(orc, x, ss, False)


def test_e2m1_exhaustive_fp16(orc):
    # Every finite fp16 value in [-6, 6] through the E2M1 conversion: blocks
    # [6, x1..x15] with tensor scale 1 get block scale 1.0, so code = E2M1(x).
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16).astype(np.float32)
    vals = f[np.isfinite(f) & (np.abs(f) <= 6.0)]
    pad = (-len(vals)) % 15
    vals = np.concatenate([vals, np.zeros(pad, np.float32)]).reshape(-1, 15)
    blocks = np.concatenate([np.full((vals.shape[0], 1), 6.0, np.float32), vals], 1)
    x = torch.from_numpy(blocks.reshape(-1, 16).astype(np.float16))
    _check_rows(orc, x, False, False, g=1.0)


def test_ue4m3_sweep(orc):
    # Block scale = UE4M3(amax / 6) with g = 1/6: one varying element per
    # block sweeps the scale conversion over fp16 magnitudes.
    h = np.arange(0, 0x7C00, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16).astype(np.float32)
    f = f[f <= 448.0]
    blocks = np.zeros((len(f), 16), np.float32)
    blocks[:, 3] = f
    blocks[:, 7] = -0.5 * f
    x = torch.from_numpy(blocks.astype(np.float16))
    _check_rows(orc, x, False, False, g=float(np.float32(1.0 / 6.0)))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("ss", [False, True])
def test_colblocks_parity(orc, dtype, ss):
    x = synth.randn16((400, 96), dtype, seed=11)
    codes, scales, ts = ops.nvfp4_quantize_colblocks(x.cuda(), use_scalesearch=ss)
    c0, s0, g0, _ = orc.nvfp4_quantize_colblocks(synth.as_u16(x), _dt(dtype), use_ss=ss)
    assert ts.item() == np.float32(g0)
    assert np.array_equal(scales.cpu().numpy(), s0)
    assert np.array_equal(codes.cpu().numpy(), c0)


def test_empty_rows():
    x = torch.zeros((0, 128), dtype=torch.float16, device="cuda")
    codes, scales, ts = ops.nvfp4_quantize(x)
    assert codes.shape == (0, 64)


def test_two_pass_path_large_tensor(orc):
    # 2^21 x 16 = 33.5M elements exceeds one resident grid of the single-pass
    # kernel, so the absmax pass and the quantise pass run separately.
    x = synth.randn16((1 << 21, 16), torch.bfloat16, seed=21)
    _check_rows(orc, x, False, False)


@pytest.mark.parametrize("had", [False, True])
@pytest.mark.parametrize("fill", [0x00, 0x5A, 0xFF])
def test_one_pass_any_workspace_contents(orc, had, fill):
    # The one-pass kernel (tensor staged in shared memory, one grid-wide max
    # exchange) counts arrivals in the caller's workspace.  The counter is
    # cleared on the stream before each launch, so a workspace full of
    # leftovers (non-zero counters, stale per-CTA maxima) still gives
    # bit-exact codes, call after call on the same buffer.
    ws = torch.full((ops.lib().nvfp4_quantize_workspace_size(),), fill, dtype=torch.uint8,
                    device="cuda")
    for seed in (11, 12, 13):
        x = synth.randn16((4096, 128), torch.bfloat16, seed=seed, scale=2.0)
        codes, scales, ts = ops.nvfp4_quantize(x.cuda(), use_hadamard=had, workspace=ws)
        torch.cuda.synchronize()
        assert ops.stream_status() == ops.OK
        c0, s0, g0, _ = orc.nvfp4_quantize(synth.as_u16(x), _dt(x.dtype), use_had=had)
        assert ts.item() == np.float32(g0)
        assert np.array_equal(scales.cpu().numpy(), s0)
        assert np.array_equal(codes.cpu().numpy(), c0)
        ws[:8].fill_(fill)  # leftovers again before the next call
