"""CUDA path vs the CPU oracle, element by element, at sizes the oracle runs in
seconds (several tiles plus ragged tails).  Calls go through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import api, synth
from nvfp4_bit_microscaled_b200._lib import Nvfp4Error
from tests._parity import assert_gemm_close, assert_q_equal, dev, gpu_amax, sample_pairs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_bit_microscaled_b200 import build
    build.build()
    api.read_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert api.read_device_error(clear=True) == 0


def _inputs():
    # (name, BF16 [R, C]) -- distributions of the workloads, shapes with tails
    return [
        ("tiny_x", synth.workload_inputs("tiny")[0]),
        ("act_outliers", synth.activations(256, 640, 21)),
        ("grad_lognormal", synth.gradients(272, 320, 22)),
        ("heavy_t3", synth.heavy_activations(144, 192, 23)),
        ("weights", synth.weights(208, 336, 24, std=0.02, outlier_frac=1e-3)),
    ]


# ------------------------------------------------------------------ amax
@pytest.mark.parametrize("shape", [(37, 48), (64, 20), (512, 1024), (3, 8)])
def test_amax_exact(shape):
    x = synth.normal(*shape, seed=5, std=3.0)
    assert gpu_amax(x) == O.amax(x)


def test_amax_strided_rows():
    big = synth.normal(40, 96, seed=6)
    view = big[:, 16:80]
    a = api.amax(dev(big)[:, 16:80])
    assert float(a.cpu()[0]) == O.amax(view.contiguous())


def test_amax_zero_tensor():
    x = torch.zeros(32, 64, dtype=torch.bfloat16)
    assert gpu_amax(x) == 0.0 and gpu_amax(x, rht=True) == 0.0


@pytest.mark.parametrize("name,x", _inputs())
def test_amax_rht_exact(name, x):
    R = x.shape[0] // 16 * 16
    x = x[:R].contiguous()
    assert gpu_amax(x, rht=True) == O.amax_rht(x), name
    both = api.amax(dev(x), rht=2).cpu().numpy()
    assert both[0] == O.amax(x) and both[1] == O.amax_rht(x), name


def test_amax_rht_narrow_columns():
    x = synth.activations(48, 12, 33)            # C % 4 == 0 but C % 8 != 0
    assert gpu_amax(x, rht=True) == O.amax_rht(x)


# ------------------------------------------------------------------ row-wise
@pytest.mark.parametrize("name,x", _inputs())
@pytest.mark.parametrize("sr", [False, True])
def test_quantize_row(name, x, sr):
    a = O.amax(x)
    amax_dev = api.amax(dev(x))
    row, _ = api.quantize(dev(x), api.ROW, amax_dev, sr=sr, seed=1234)
    codes, sf = O.quantize_row(x, a, sr=sr, seed=1234)
    assert_q_equal(row, codes, sf, a, f"{name} row sr={sr}")


def test_quantize_row_partial_scale_word_and_row_padding():
    x = synth.activations(131, 48, 31)        # S = 3: one partial scale word; 131 rows: padding
    a = O.amax(x)
    row, _ = api.quantize(dev(x), api.ROW, api.amax(dev(x)))
    assert_q_equal(row, *O.quantize_row(x, a), a, "ragged row")


def test_quantize_row_ties_and_saturation():
    # Scaled values exactly on E2M1 midpoints and above 6: S_enc = 1 (amax 2688),
    # blocks whose max is 6 get scale 1, so y = x exactly.
    vals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -5.0, -0.0, 0.1, -0.1, 6.0, 4.0]
    x = np.zeros((2, 64), dtype=np.float32)
    x[0, 0] = 2688.0
    for b in range(1, 4):
        x[0, 16 * b] = 6.0
        x[0, 16 * b + 1:16 * b + 16] = vals
    x[1, :16] = np.linspace(-7, 7, 16)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    a = O.amax(xb)
    row, _ = api.quantize(dev(xb), api.ROW, api.amax(dev(xb)))
    assert_q_equal(row, *O.quantize_row(xb, a), a, "ties")


def test_quantize_row_sr_distribution_matches_worked_example():
    # y = 3.4 (bf16 3.40625) with scale 1: P(4) ~ 0.40625 over many elements
    n_blocks = 4096
    x = np.full((1, 16 * n_blocks), 3.40625, dtype=np.float32)
    x[0, 0::16] = 6.0
    x[0, 0] = 2688.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    row, _ = api.quantize(dev(xb), api.ROW, api.amax(dev(xb)), sr=True, seed=99)
    data = row.data.cpu().numpy()[0]
    codes = np.empty(data.size * 2, dtype=np.uint8)
    codes[0::2], codes[1::2] = data & 15, data >> 4
    sel = np.ones(codes.size, bool)
    sel[0::16] = False
    sel[:16] = False                           # block 0 holds the tensor max and scales differently
    up = np.mean(codes[sel] == 0x6)            # code 6 = 4.0, code 5 = 3.0
    assert set(np.unique(codes[sel])) <= {5, 6}
    assert abs(up - 0.40625) < 5 * 0.5 / np.sqrt(sel.sum())


def _grid_blocks(rows, blocks_per_row):
    # every 16-element block: max 6 * 2^k (so its E4M3 scale is exactly 2^k with S_enc = 1) and
    # values on the E2M1 grid, on its binade boundaries and at its midpoints, with random signs;
    # one element of 2688 fixes the tensor amax (S_enc = 2688 / 2688 = 1)
    vals = np.array([6.0, 4.0, 3.0, 2.0, 1.5, 1.0, 0.5, 0.0, 5.0, 3.5, 2.5, 1.75, 1.25, 0.75, 0.25, 0.125],
                    dtype=np.float32)
    rng = np.random.default_rng(11)
    x = np.empty((rows, 16 * blocks_per_row), dtype=np.float32)
    for r in range(rows):
        for b in range(blocks_per_row):
            k = rng.integers(-6, 7)
            blk = rng.permutation(vals) * np.float32(2.0 ** k)
            blk[np.argmax(np.abs(blk))] = np.float32(6.0 * 2.0 ** k)
            x[r, 16 * b:16 * b + 16] = blk * rng.choice(np.array([-1.0, 1.0], dtype=np.float32), 16)
    x[0, 0] = 2688.0
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("seed", [1, 12345])
def test_sr_on_grid_points_boundaries_and_midpoints(seed):
    # the SR decision's directed roundings (fma.rp / add.rp on FP32 pairs) at the values where
    # they matter: scaled values exactly on the grid (must not move), on the binade boundaries
    # 1, 2, 4, 6 and at midpoints; row and column copies, bit-exact against the oracle
    xb = _grid_blocks(64, 20)
    a = O.amax(xb)
    assert a == 2688.0
    row, _ = api.quantize(dev(xb), api.ROW, api.amax(dev(xb)), sr=True, seed=seed)
    assert_q_equal(row, *O.quantize_row(xb, a, sr=True, seed=seed), a, "row SR on grid values")
    xt = xb.t().contiguous()      # the same blocks down the columns
    at = O.amax(xt)
    _, col = api.quantize(dev(xt), api.COL, api.amax(dev(xt)), sr=True, seed=seed)
    assert_q_equal(col, *O.quantize_col(xt, at, sr=True, seed=seed), at, "column SR on grid values")
    # values already on the grid come back unchanged, whatever the random words
    data = row.data.cpu().numpy()
    codes = np.empty((data.shape[0], data.shape[1] * 2), dtype=np.uint8)
    codes[:, 0::2], codes[:, 1::2] = data & 15, data >> 4
    cr, _ = O.quantize_row(xb, a)          # round to nearest: exact on grid values
    on_grid = np.isin(np.abs(xb.float().numpy()) / np.repeat(
        np.maximum(np.abs(xb.float().numpy()).reshape(64, -1, 16).max(axis=2), 1e-30) / 6.0, 16, axis=1),
        [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    on_grid[0, :16] = False                # block 0 holds the tensor max
    assert np.array_equal(codes[on_grid], np.asarray(cr)[on_grid])


# ------------------------------------------------------------------ column-wise
@pytest.mark.parametrize("name,x", _inputs())
@pytest.mark.parametrize("rht,sr", [(False, False), (True, False), (False, True), (True, True)])
def test_quantize_col(name, x, rht, sr):
    R = x.shape[0] // 16 * 16
    x = x[:R].contiguous()
    if x.shape[1] % 8:
        pytest.skip("column path needs C % 4 == 0 and the RHT amax C % 8 == 0")
    a = O.amax_rht(x) if rht else O.amax(x)
    amax_dev = api.amax(dev(x), rht=rht)
    assert float(amax_dev.cpu()[0]) == a
    _, col = api.quantize(dev(x), api.COL, amax_dev, rht=rht, sr=sr, seed=77)
    codes, sf = O.quantize_col(x, a, rht=rht, sr=sr, seed=77)
    assert_q_equal(col, codes, sf, a, f"{name} col rht={rht} sr={sr}")


@pytest.mark.parametrize("R,C", [(48, 100), (32, 4), (48, 1028), (80, 1540)])
@pytest.mark.parametrize("rht,sr", [(False, False), (True, False), (False, True), (True, True)])
def test_quantize_col_four_channel_tail(R, C, rht, sr):
    # C % 8 == 4: a strip's last four channels are not a whole 16-byte copy and
    # are read from global memory; with C = 4, 1028 and 1540 the last
    # 512-channel strip has nothing to copy at all.  The amax is the oracle's,
    # passed in (the device RHT amax wants C % 8 == 0).
    # rows padded to C + 4 channels: the row stride must be a multiple of 8
    x = synth.gradients(R, C, 51)
    a = O.amax_rht(x) if rht else O.amax(x)
    amax_dev = torch.tensor([a], dtype=torch.float32, device="cuda")
    xp = torch.zeros(R, C + 4, dtype=torch.bfloat16, device="cuda")
    xp[:, :C] = dev(x)
    _, col = api.quantize(xp[:, :C], api.COL, amax_dev, rht=rht, sr=sr, seed=78)
    codes, sf = O.quantize_col(x, a, rht=rht, sr=sr, seed=78)
    assert_q_equal(col, codes, sf, a, f"col tail {R}x{C} rht={rht} sr={sr}")


@pytest.mark.parametrize("rht,sr", [(False, False), (True, False), (False, True), (True, True)])
def test_quantize_col_strided_rows(rht, sr):
    # a row stride past C: the staged copies read each row from its own stride
    big = synth.gradients(96, 776, 53)
    x = dev(big)[:, :768]
    xc = big[:, :768].contiguous()
    a = O.amax_rht(xc) if rht else O.amax(xc)
    _, col = api.quantize(x, api.COL, api.amax(x, rht=rht), rht=rht, sr=sr, seed=79)
    codes, sf = O.quantize_col(xc, a, rht=rht, sr=sr, seed=79)
    assert_q_equal(col, codes, sf, a, f"col strided rht={rht} sr={sr}")


@pytest.mark.parametrize("rht,sr", [(True, True), (True, False), (False, True)])
def test_quantize_col_many_items_per_cta(rht, sr):
    # 8192 tokens x 1600 channels: 2048 items of 16 tokens x a 512-channel
    # strip (the last strip 64 channels), more than three per resident CTA, so
    # every stage buffer is refilled and its barrier runs through both phases
    x = synth.gradients(8192, 1600, 54)
    a = O.amax_rht(x) if rht else O.amax(x)
    _, col = api.quantize(dev(x), api.COL, api.amax(dev(x), rht=rht), rht=rht, sr=sr, seed=80)
    codes, sf = O.quantize_col(x, a, rht=rht, sr=sr, seed=80)
    assert_q_equal(col, codes, sf, a, f"col 8192x1600 rht={rht} sr={sr}")


@pytest.mark.parametrize("rht", [False, True])
def test_quantize_rowcol_many_items_per_cta(rht):
    x = synth.activations(8192, 1600, 55)
    a, ar = O.amax(x), O.amax_rht(x)
    amax_dev = api.amax(dev(x), rht=2) if rht else api.amax(dev(x))
    row, col = api.quantize(dev(x), api.ROWCOL, amax_dev, rht=rht)
    assert_q_equal(row, *O.quantize_row(x, a), a, "rowcol 8192x1600 row")
    ac = ar if rht else a
    assert_q_equal(col, *O.quantize_col(x, ac, rht=rht), ac, f"rowcol 8192x1600 col rht={rht}")


def test_quantize_rowcol():
    x = synth.gradients(192, 256, 41)
    a = O.amax(x)
    row, col = api.quantize(dev(x), api.ROWCOL, api.amax(dev(x)), sr=True, seed=5)
    assert_q_equal(row, *O.quantize_row(x, a, sr=True, seed=5), a, "rowcol row")
    assert_q_equal(col, *O.quantize_col(x, a, sr=True, seed=5), a, "rowcol col")


@pytest.mark.parametrize("name,x", _inputs())
@pytest.mark.parametrize("rht", [False, True])
def test_quantize_rowcol_one_read(name, x, rht):
    # ROWCOL without SR: one kernel writes both copies from one read of x; with
    # RHT the column copy is the RHT copy, scaled by the RHT amax (amax_dev[1])
    R = x.shape[0] // 16 * 16
    x = x[:R].contiguous()
    a, ar = O.amax(x), O.amax_rht(x)
    amax_dev = api.amax(dev(x), rht=2) if rht else api.amax(dev(x))
    row, col = api.quantize(dev(x), api.ROWCOL, amax_dev, rht=rht)
    assert_q_equal(row, *O.quantize_row(x, a), a, f"{name} rowcol row")
    ac = ar if rht else a
    assert_q_equal(col, *O.quantize_col(x, ac, rht=rht), ac, f"{name} rowcol col rht={rht}")


@pytest.mark.parametrize("R,C", [(64, 128), (80, 144), (16, 4096 + 16), (1040, 272)])
def test_quantize_rowcol_one_read_tails(R, C):
    # token counts that are not multiples of 64 and channel counts that are not multiples of 128
    x = synth.activations(R, C, 44)
    a, ar = O.amax(x), O.amax_rht(x)
    row, col = api.quantize(dev(x), api.ROWCOL, api.amax(dev(x), rht=2), rht=True)
    assert_q_equal(row, *O.quantize_row(x, a), a, f"rowcol row {R}x{C}")
    assert_q_equal(col, *O.quantize_col(x, ar, rht=True), ar, f"rowcol col {R}x{C}")


# ------------------------------------------------------------------ 2D
@pytest.mark.parametrize("shape", [(128, 256), (48, 80), (208, 336), (16, 16)])
def test_quantize_2d(shape):
    w = synth.weights(*shape, seed=51, std=0.02, outlier_frac=2e-3)
    a = O.amax(w)
    row, col = api.quantize(dev(w), api.TWO_D, api.amax(dev(w)))
    codes, sft = O.quantize_2d(w, a)
    (rc, rs), (cc, cs) = O.expand_2d(codes, sft)
    assert_q_equal(row, rc, rs, a, f"2d row {shape}")
    assert_q_equal(col, cc, cs, a, f"2d col {shape}")


def test_2d_column_copy_equals_2d_of_transpose():
    w = synth.weights(96, 160, 52, std=1.0)
    wt = w.T.contiguous()
    amax_dev = api.amax(dev(w))
    _, col = api.quantize(dev(w), api.TWO_D, amax_dev, row_out=False)
    row_t, _ = api.quantize(dev(wt), api.TWO_D, amax_dev, col_out=False)
    assert torch.equal(col.data, row_t.data) and torch.equal(col.scales, row_t.scales)


# ------------------------------------------------------------------ GEMM
def _qrow(x, sr=False, seed=0):
    a = O.amax(x)
    q, _ = api.quantize(dev(x), api.ROW, api.amax(dev(x)), sr=sr, seed=seed)
    codes, sf = O.quantize_row(x, a, sr=sr, seed=seed)
    assert_q_equal(q, codes, sf, a, "gemm operand")
    return q, codes, sf, float(O.global_scales(a)[1])


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 512, 512), (200, 272, 320), (384, 256, 1024),
                                   (130, 48, 64), (1000, 1040, 320), (520, 20480 + 16, 64), (96, 400, 256)])
@pytest.mark.parametrize("bf16", [False, True])
def test_gemm_full_vs_oracle(M, N, K, bf16):
    xa = synth.activations(M, K, 61)
    xb = synth.weights(N, K, 62, std=0.02)
    qa, ca, sa, ga = _qrow(xa)
    qb, cb, sb, gb = _qrow(xb)
    D = api.gemm(qa, qb, api.OUT_BF16 if bf16 else api.OUT_F32)
    D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
    assert_gemm_close(D.float().cpu().numpy(), D_ref, absum, bf16=bf16, what=f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (512, 768, 1280), (1024, 2048, 64), (768, 512, 320),
                                   (2304, 1536, 512)])
@pytest.mark.parametrize("bf16", [False, True])
def test_gemm_cta_pair_path_vs_oracle(M, N, K, bf16):
    # more than 128 rows: the CTA-pair kernel (cta_group::2)
    xa = synth.activations(M, K, 63)
    xb = synth.weights(N, K, 64, std=0.02)
    qa, ca, sa, ga = _qrow(xa)
    qb, cb, sb, gb = _qrow(xb)
    D = api.gemm(qa, qb, api.OUT_BF16 if bf16 else api.OUT_F32)
    if M * N <= 1 << 20:
        D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
        assert_gemm_close(D.float().cpu().numpy(), D_ref, absum, bf16=bf16, what=f"pair {M}x{N}x{K}")
    else:
        pairs = sample_pairs(M, N, 8192, seed=5)
        D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb, pairs=pairs)
        Dn = D.float().cpu().numpy()
        assert_gemm_close(Dn[pairs[:, 0], pairs[:, 1]], D_ref, absum, bf16=bf16, what=f"pair {M}x{N}x{K}")


@pytest.mark.parametrize("pad", [8, 24])
@pytest.mark.parametrize("bf16", [False, True])
def test_gemm_output_row_stride(pad, bf16):
    # D written into a wider buffer (row stride N + pad) by the CTA-pair
    # kernel's TMA-store epilogue; the columns past N stay untouched.
    M, N, K = 512, 256, 320
    xa = synth.activations(M, K, 65)
    xb = synth.weights(N, K, 66, std=0.02)
    qa, ca, sa, ga = _qrow(xa)
    qb, cb, sb, gb = _qrow(xb)
    dt = torch.bfloat16 if bf16 else torch.float32
    buf = torch.full((M, N + pad), 7.0, dtype=dt, device="cuda")
    api.gemm(qa, qb, api.OUT_BF16 if bf16 else api.OUT_F32, out=buf[:, :N])
    D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
    got = buf.float().cpu().numpy()
    assert_gemm_close(got[:, :N], D_ref, absum, bf16=bf16, what=f"ldd {N + pad}")
    assert (got[:, N:] == 7.0).all()


def test_gemm_rejects_unaligned_row_stride_before_launch():
    M, N, K = 256, 256, 64
    qa, _, _, _ = _qrow(synth.activations(M, K, 67))
    qb, _, _, _ = _qrow(synth.weights(N, K, 68, std=0.02))
    buf = torch.zeros((M, N + 3), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Nvfp4Error) as e:
        api.gemm(qa, qb, api.OUT_BF16, out=buf[:, :N])
    assert e.value.status == 3  # NVFP4_ERR_ALIGN
    assert (buf == 0).all()


@pytest.mark.parametrize("M,N,K", [(256, 256, 96), (512, 256, 160), (256, 512, 288), (200, 272, 96),
                                   (130, 48, 160),                                           # CTA-pair kernel
                                   (128, 272, 96), (72, 48, 160)])                           # single-CTA kernel
@pytest.mark.parametrize("bf16", [False, True])
def test_gemm_k_tail_of_32(M, N, K, bf16):
    # K % 64 == 32: the last K=64 step is completed with zero codes (TMA fill
    # past the row) and zero scales (scale-matrix padding)
    xa = synth.activations(M, K, 81)
    xb = synth.weights(N, K, 82, std=0.02)
    qa, ca, sa, ga = _qrow(xa)
    qb, cb, sb, gb = _qrow(xb)
    D = api.gemm(qa, qb, api.OUT_BF16 if bf16 else api.OUT_F32)
    D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
    assert_gemm_close(D.float().cpu().numpy(), D_ref, absum, bf16=bf16, what=f"K tail {M}x{N}x{K}")


def test_gemm_tiny_workload():
    x, w, _ = synth.workload_inputs("tiny")
    qa, ca, sa, ga = _qrow(x)
    qb, cb, sb, gb = _qrow(w)
    D = api.gemm(qa, qb)
    D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
    assert_gemm_close(D.cpu().numpy(), D_ref, absum, what="tiny")


def _handmade_operand(codes, sf_byte=0x38):
    """A QTensor built on the host from explicit codes and one scale value (1.0)."""
    R, K = codes.shape
    data = torch.from_numpy(O.pack_nibbles(codes))
    sf = O.swizzle_scales(np.full((R, K // 16), sf_byte, np.uint8))
    return api.QTensor(data.cuda(), torch.from_numpy(sf).cuda(), torch.ones(1, device="cuda"), R, K)


def test_gemm_one_hot_pins_nibble_order_and_scale_layout():
    # A[0, 1] = 1.0 (code 2) and B row n holds value n-dependent codes: D[0, n] = B[n, 1]
    M, N, K = 128, 256, 256
    ca = np.zeros((M, K), np.uint8)
    ca[0, 1] = 0x2
    ca[5, 130] = 0x7                           # 6.0 at k = 130 (second MMA step of the tile)
    rng = np.random.default_rng(0)
    cb = rng.integers(0, 16, (N, K)).astype(np.uint8)
    A, B = _handmade_operand(ca), _handmade_operand(cb)
    D = api.gemm(A, B).cpu().numpy()
    val = np.array([O.e2m1_decode(c) for c in range(16)])
    assert np.array_equal(D[0], val[cb[:, 1]])
    assert np.array_equal(D[5], 6.0 * val[cb[:, 130]])
    assert not D[1:5].any()
    # one distinct scale per (row, block): exercises every byte of the 128x4 tile layout
    sfa = rng.integers(0x30, 0x40, (M, K // 16)).astype(np.uint8)
    sfb = rng.integers(0x30, 0x40, (N, K // 16)).astype(np.uint8)
    ca2 = rng.integers(0, 16, (M, K)).astype(np.uint8)
    A2 = api.QTensor(torch.from_numpy(O.pack_nibbles(ca2)).cuda(), torch.from_numpy(O.swizzle_scales(sfa)).cuda(),
                     torch.ones(1, device="cuda"), M, K)
    B2 = api.QTensor(torch.from_numpy(O.pack_nibbles(cb)).cuda(), torch.from_numpy(O.swizzle_scales(sfb)).cuda(),
                     torch.ones(1, device="cuda"), N, K)
    D2 = api.gemm(A2, B2).cpu().numpy()
    D_ref, absum = O.gemm(ca2, sfa, 1.0, cb, sfb, 1.0)
    assert_gemm_close(D2, D_ref, absum, what="scale layout")


def test_gemm_global_scales_applied():
    x = synth.normal(128, 256, 71, std=0.001)
    w = synth.normal(256, 256, 72, std=50.0)
    qa, ca, sa, ga = _qrow(x)
    qb, cb, sb, gb = _qrow(w)
    D = api.gemm(qa, qb).cpu().numpy()
    D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
    assert_gemm_close(D, D_ref, absum, what="global scales")


def test_gemm_sampled_multi_wave():
    # more tiles than SMs: exercises the persistent schedule and stage reuse
    M, N, K = 2048, 4096, 768
    xa = synth.activations(M, K, 81)
    xb = synth.weights(N, K, 82, std=0.02)
    qa, ca, sa, ga = _qrow(xa)
    qb, cb, sb, gb = _qrow(xb)
    D = api.gemm(qa, qb).cpu().numpy()
    pairs = sample_pairs(M, N, 4096, seed=3)
    D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb, pairs=pairs)
    assert_gemm_close(D[pairs[:, 0], pairs[:, 1]], D_ref, absum, what="multi-wave")


# ------------------------------------------------------------------ linear layer
def test_linear_fwd_bwd_vs_oracle():
    T, Cin, Cout, seed = 256, 320, 384, 2024
    X = synth.activations(T, Cin, 91)
    W = synth.weights(Cout, Cin, 92)
    dY = synth.gradients(T, Cout, 93)
    ws = api.LinearWorkspace(T, Cin, Cout, "cuda")
    Y = api.linear_fwd(dev(X), dev(W), ws)
    dX, dW = api.linear_bwd(dev(dY), ws, seed)
    torch.cuda.synchronize()
    # oracle, step by step in the layer's order
    ax, aw, axr = O.amax(X), O.amax(W), O.amax_rht(X)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), (cwc, swc) = O.expand_2d(cw, tw)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    ag, agr = O.amax(dY), O.amax_rht(dY)
    cg, sg = O.quantize_row(dY, ag, sr=True, seed=seed)
    cgc, sgc = O.quantize_col(dY, agr, rht=True, sr=True, seed=seed)
    gs = lambda a: float(O.global_scales(a)[1])
    assert_q_equal(ws.tensor("x_row"), cx, sx, ax, "x_row")
    assert_q_equal(ws.tensor("w_row"), cwr, swr, aw, "w_row")
    assert_q_equal(ws.tensor("w_col"), cwc, swc, aw, "w_col")
    assert_q_equal(ws.tensor("x_col"), cxc, sxc, axr, "x_col")
    assert_q_equal(ws.tensor("dy_row"), cg, sg, ag, "dy_row")
    assert_q_equal(ws.tensor("dy_col"), cgc, sgc, agr, "dy_col")
    Yr, Ya = O.gemm(cx, sx, gs(ax), cwr, swr, gs(aw))
    assert_gemm_close(Y.float().cpu().numpy(), Yr, Ya, bf16=True, what="Y")
    dXr, dXa = O.gemm(cg, sg, gs(ag), cwc, swc, gs(aw))
    assert_gemm_close(dX.float().cpu().numpy(), dXr, dXa, bf16=True, what="dX")
    dWr, dWa = O.gemm(cgc, sgc, gs(agr), cxc, sxc, gs(axr))
    assert_gemm_close(dW.cpu().numpy(), dWr, dWa, what="dW")


# ------------------------------------------------------------------ bounded waits
def test_block_scale_division_matches_ieee_on_every_float():
    # the kernels divide by 6 with a corrected reciprocal product; every
    # non-negative float gives the IEEE quotient where it is normal, and the
    # same E4M3 scale code everywhere
    assert api.selftest_scale_division() == (0, 0)


def test_sr_conversion_follows_the_rounding_rule_for_every_draw():
    # the SR quantizers round with the hardware conversion: every 16-bit draw
    # of every lane, for 8192 values over [0, 6.5), rounds up exactly when
    # draw + floor(p * 2^16) >= 2^16 (the oracle's R10)
    mismatches, checked = api.selftest_sr_rounding()
    assert checked == 8192 * 4 * 65536
    assert mismatches == 0


def test_wait_probe_times_out_and_reports():
    api.read_device_error(clear=True)
    api.wait_probe(20000)                      # 20 ms; nothing ever arrives
    torch.cuda.synchronize()
    assert api.read_device_error(clear=True) == 5
    assert api.read_device_error(clear=True) == 0
    # the context is still usable afterwards
    x = synth.normal(64, 64, 1)
    assert gpu_amax(x) == O.amax(x)


# ------------------------------------------------------------------ GEMM with epilogue amax
@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (96, 48, 128), (128, 272, 96),       # single-CTA kernel
                                   (256, 256, 256), (200, 272, 320), (1000, 528, 256),   # CTA pairs, M/N tails
                                   (2304, 1536, 512)])
@pytest.mark.parametrize("bf16", [False, True])
def test_gemm_amax_is_max_of_stored_output(M, N, K, bf16):
    xa = synth.activations(M, K, 91)
    xb = synth.weights(N, K, 92, std=0.02)
    qa, ca, sa, ga = _qrow(xa)
    qb, cb, sb, gb = _qrow(xb)
    out = api.OUT_BF16 if bf16 else api.OUT_F32
    amax_buf = torch.full((1,), 1e30, dtype=torch.float32, device="cuda")   # must be overwritten
    D, amax = api.gemm_amax(qa, qb, out, amax_out=amax_buf)
    D_plain = api.gemm(qa, qb, out)
    assert torch.equal(D, D_plain)                            # same outputs as nvfp4_gemm
    got = float(amax.cpu()[0])
    assert got == float(D.float().abs().max().cpu())          # exactly the max of what was stored
    if bf16:
        assert got == float(api.amax(D).cpu()[0])             # the value the amax pass would give
    if M * N <= 1 << 20:
        D_ref, absum = O.gemm(ca, sa, ga, cb, sb, gb)
        assert_gemm_close(D.float().cpu().numpy(), D_ref, absum, bf16=bf16, what=f"gemm_amax {M}x{N}x{K}")
        # and within the GEMM tolerance of the oracle's own max |D|
        tol = 1e-4 * absum + (2.0 ** -8 * np.abs(D_ref) if bf16 else 0.0)
        assert got <= np.max(np.abs(D_ref) + tol) and got >= np.max(np.abs(D_ref) - tol)


def test_gemm_amax_zero_operand_and_reuse():
    M, N, K = 256, 256, 128
    qa, _, _, _ = _qrow(torch.zeros(M, K, dtype=torch.bfloat16))
    qb, _, _, _ = _qrow(synth.weights(N, K, 93, std=0.02))
    amax_buf = torch.full((1,), 5.0, dtype=torch.float32, device="cuda")
    D, amax = api.gemm_amax(qa, qb, api.OUT_BF16, amax_out=amax_buf)
    assert float(amax.cpu()[0]) == 0.0 and not D.any()
    qa2, _, _, _ = _qrow(synth.activations(M, K, 94))
    D2, amax2 = api.gemm_amax(qa2, qb, api.OUT_BF16, amax_out=amax_buf)   # same buffer, zeroed again
    assert float(amax2.cpu()[0]) == float(D2.float().abs().max().cpu()) > 0.0


def test_gemm_amax_feeds_the_next_quantize():
    # the fused amax replaces the amax pass in front of quantizing D
    M, N, K = 512, 768, 256
    qa, _, _, _ = _qrow(synth.activations(M, K, 95))
    qb, _, _, _ = _qrow(synth.weights(N, K, 96, std=0.02))
    D, amax = api.gemm_amax(qa, qb, api.OUT_BF16)
    q_fused, _ = api.quantize(D, api.ROW, amax)
    q_pass, _ = api.quantize(D, api.ROW, api.amax(D))
    assert torch.equal(q_fused.data, q_pass.data) and torch.equal(q_fused.scales, q_pass.scales)
    assert torch.equal(q_fused.global_scale, q_pass.global_scale)
