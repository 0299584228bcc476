"""Pins of the oracle's MXFP4 functions (readings R21-R24: 1x32 blocks, UE8M0
scales, OCP Microscaling scale rule), each against something other than the
oracle itself: torch's own UE8M0 dtype, numpy's log2, values worked by hand on
the E2M1 grid, exact round trips, and numpy matmuls.  CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import synth

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def test_e8m0_decode_matches_torch_float8_e8m0fnu():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = np.array([O.e8m0_decode(b) for b in range(256)])
    assert np.isnan(got[255]) and np.isnan(ref[255])
    assert np.array_equal(got[:255], ref[:255])
    assert got[127] == 1.0 and got[0] == 2.0 ** -127 and got[254] == 2.0 ** 127


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_scale_exponent_matches_numpy_log2(seed):
    rng = np.random.default_rng(seed)
    vals = np.exp2(rng.uniform(-120, 120, 2000)).astype(np.float32)
    vals = _bf16(vals).float().numpy()                       # values a BF16 tensor can hold
    for v in vals:
        s = O.mx_scale_exponent(v)
        assert s == int(np.floor(np.log2(np.float64(v)))) - 2, v
    assert O.mx_scale_exponent(0.0) == -127                   # all-zero block
    assert O.mx_scale_exponent(2.0 ** -133) == -127           # clamped below
    assert O.mx_scale_exponent(1.5 * 2.0 ** 127) == 125


def test_scaled_block_max_lies_in_four_to_eight():
    # the OCP rule puts the block maximum at [4, 8) times the scale, so only
    # values >= 6 * 2^s saturate
    x = synth.activations(64, 256, 7)
    codes, sf = O.mx_quantize_row(x)
    xf = x.float().numpy().reshape(64, 8, 32)
    bamax = np.abs(xf).max(axis=2)
    scale = np.exp2(sf.astype(np.float64) - 127)
    ratio = bamax / scale
    assert ((ratio >= 4) & (ratio < 8)).all()


@pytest.mark.parametrize("k", [-120, -9, 0, 5, 100])
def test_exact_round_trip_for_grid_blocks(k):
    rng = np.random.default_rng(k + 200)
    c = rng.choice(np.array(GRID + [-g for g in GRID[1:]]), size=(4, 64))
    c[:, 0] = 6.0
    c[:, 32] = -6.0
    x = _bf16(c * 2.0 ** k)
    codes, sf = O.mx_quantize_row(x)
    assert (sf == 127 + k).all()
    assert np.array_equal(O.mx_dequantize(codes, sf), x.double().numpy())


def test_worked_block_saturation_and_ties():
    # scale 2^0 (block max 7: floor(log2 7) - 2 = 0); 7 saturates to 6; the
    # midpoints go to the even grid index: 3.5 -> 4, 2.5 -> 2, 0.75 -> 1, 0.25 -> 0
    vals = [7.0, 3.5, 2.5, 0.75, 0.25, -5.0, -0.25, 1.25] + [0.0] * 24
    codes, sf = O.mx_quantize_row(_bf16([vals]))
    assert sf[0, 0] == 127
    want_mag = [6.0, 4.0, 2.0, 1.0, 0.0, 4.0, 0.0, 1.0]
    want_sign = [0, 0, 0, 0, 0, 1, 0, 0]
    for i, (m, sg) in enumerate(zip(want_mag, want_sign)):
        code = codes[0, i]
        assert GRID[code & 7] == m, (i, code)
        assert (code >> 3) == (sg if m != 0.0 else 0), (i, code)   # zero is always +0 (R2)


def test_mx_gemm_integer_case_is_exact():
    rng = np.random.default_rng(3)
    M, N, K = 24, 40, 96
    ca = rng.integers(0, 16, (M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, (N, K), dtype=np.uint8)
    sa = np.full((M, K // 32), 127, np.uint8)
    sb = np.full((N, K // 32), 128, np.uint8)                # scale 2
    D, absum = O.mx_gemm(ca, sa, cb, sb)
    g = np.array(GRID + [-v for v in GRID])
    g[8] = 0.0                                                # code 8 is -0
    ref = (g[ca] @ (2.0 * g[cb]).T)
    assert np.array_equal(D, ref)
    assert np.array_equal(absum, np.abs(g[ca]) @ np.abs(2.0 * g[cb]).T)


def test_mx_gemm_matches_numpy_on_quantized_operands():
    xa = synth.activations(48, 128, 8)
    xb = synth.weights(40, 128, 9, std=0.02)
    ca, sa = O.mx_quantize_row(xa)
    cb, sb = O.mx_quantize_row(xb)
    D, _ = O.mx_gemm(ca, sa, cb, sb)
    ref = O.mx_dequantize(ca, sa) @ O.mx_dequantize(cb, sb).T
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-30)
    pairs = np.array([[0, 0], [47, 39], [13, 7]], dtype=np.int64)
    Dp, _ = O.mx_gemm(ca, sa, cb, sb, pairs=pairs)
    assert np.array_equal(Dp, D[pairs[:, 0], pairs[:, 1]])


@pytest.mark.parametrize("name", ["activations", "weights", "gradients"])
def test_nvfp4_round_trip_error_below_mxfp4(name):
    # the pages' comparison (section 2A): 16-element blocks with E4M3 scales
    # represent the same tensors more accurately than 32-element UE8M0 blocks
    x = {"activations": lambda: synth.activations(256, 512, 10),
         "weights": lambda: synth.weights(256, 512, 11, std=0.02),
         "gradients": lambda: synth.gradients(256, 512, 12)}[name]()
    xf = x.double().numpy()
    a = O.amax(x)
    codes, sf = O.quantize_row(x, a)
    nv = O.dequantize(codes, sf, O.global_scales(a)[1])
    mc, ms = O.mx_quantize_row(x)
    mx = O.mx_dequantize(mc, ms)
    err_nv = np.sum((nv - xf) ** 2) / np.sum(xf ** 2)
    err_mx = np.sum((mx - xf) ** 2) / np.sum(xf ** 2)
    assert err_nv < err_mx, (err_nv, err_mx)
    assert math.isfinite(err_nv) and math.isfinite(err_mx)
