"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test ties one oracle function to a published value, a closed form, an
invariant, or an independent library routine, so that a dropped term, a wrong
sign or index or a transposed operand fails somewhere here.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ----------------------------------------------------------------- formats
def test_e2m1_grid_matches_published_code_points():
    for code, val in _rows("e2m1_grid.txt"):
        got = O.e2m1_decode(int(code, 16))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_named_points_and_shape():
    for code, val in _rows("e4m3_points.txt"):
        got = O.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val)
    pos = [O.e4m3_decode(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(pos, pos[1:]))        # strictly increasing
    assert len(pos) == 127 and pos[-1] == 448.0             # 126 positive finite + zero


def test_e2m1_encode_ties_and_saturation():
    # round-to-nearest-even on the midpoints: the even code wins
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for y, want in ties.items():
        assert O.e2m1_decode(O.e2m1_encode_rn(y)) == want
        assert O.e2m1_decode(O.e2m1_encode_rn(-y)) == -want
        up, dn = np.nextafter(np.float32(y), np.float32(10)), np.nextafter(np.float32(y), np.float32(-10))
        grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
        i = max(k for k, g in enumerate(grid) if g < y)
        assert O.e2m1_decode(O.e2m1_encode_rn(float(up))) == grid[i + 1]
        assert O.e2m1_decode(O.e2m1_encode_rn(float(dn))) == grid[i]
    for y in (6.0, 6.4, 7.0, 100.0, 3e38):
        assert O.e2m1_encode_rn(y) == 0x7 and O.e2m1_encode_rn(-y) == 0xF
    # a negative value that rounds to zero encodes as +0
    assert O.e2m1_encode_rn(-0.1) == 0 and O.e2m1_encode_rn(-0.0) == 0


def test_e2m1_encode_error_bound_and_monotone():
    ys = np.linspace(-7, 7, 20001, dtype=np.float32)
    vals = np.array([O.e2m1_decode(O.e2m1_encode_rn(float(y))) for y in ys])
    assert np.all(np.diff(vals) >= 0)
    a = np.abs(ys).astype(np.float64)
    half_step = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
    inside = a <= 6
    assert np.all(np.abs(vals - ys)[inside] <= half_step[inside])


def test_e4m3_encode_matches_torch_float8_cast():
    # torch's float32 -> float8_e4m3fn cast is round-to-nearest-even; below the
    # saturation region it must agree with the oracle bit for bit.
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        np.exp2(rng.uniform(-16, np.log2(463.9), 200000)).astype(np.float32),
        np.array([O.e4m3_decode(c) for c in range(1, 0x7E)], dtype=np.float32),
        # exact midpoints between neighbours (ties)
        np.array([(O.e4m3_decode(c) + O.e4m3_decode(c + 1)) / 2 for c in range(0, 0x7D)], dtype=np.float32),
        np.float32([0.0, 2.0 ** -10, 2.0 ** -11, 2.0 ** -10 * 1.0001]),
    ])
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_encode_rn_sat(float(x)) for x in xs], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_encode_saturates():
    for d in (448.0, 460.0, 464.0, 500.0, 1e6, 3e38):
        assert O.e4m3_encode_rn_sat(d) == 0x7E


# ----------------------------------------------------------------- philox
def test_philox_known_answers():
    for row in _rows("philox_kat.txt"):
        v = [int(t, 16) for t in row]
        out = O.philox4x32_10(v[0:4], v[4:6])
        assert list(out) == v[6:10]


def test_sr_block_keying():
    # R11: one generator call per 16-element block, the counter's low and high
    # words from g, its third word the domain
    seed = 0x0123456789ABCDEF
    for g in (0, 1, 2, 5, 2 ** 33 + 5):
        out = O.philox4x32_10([g & 0xFFFFFFFF, g >> 32, 1, 0], [seed & 0xFFFFFFFF, seed >> 32])
        assert list(O.sr_block_words(seed, g, 1)) == list(out)
        draws = O.sr_block_draws(seed, g, 1)
        assert [int(d) for d in draws] == [O.sr_draw16(out[i // 4], i % 4) for i in range(16)]


def _rev(x, n):
    return int(format(x, f"0{n}b")[::-1], 2)


def test_sr_draw_is_a_bijection_of_its_sixteen_bits():
    # R10: each element's draw is a bijection of the 16 bits it reads, so a
    # uniform word gives a uniform draw; the two elements that read the same 16
    # bits get them in opposite orders, and the other two bytes never enter
    for q in range(4):
        lo_byte, hi_byte = (0, 2) if q < 2 else (1, 3)
        other = [k for k in range(4) if k not in (lo_byte, hi_byte)]
        seen = np.zeros(1 << 16, dtype=np.int32)
        for lo in range(256):
            for hi in range(256):
                noise = ((lo * 7 + hi) & 0xFF) << (8 * other[0]) | ((hi * 13 + 5) & 0xFF) << (8 * other[1])
                d = O.sr_draw16((lo << (8 * lo_byte)) | (hi << (8 * hi_byte)) | noise, q)
                natural = (hi << 8) | lo
                assert d == (natural if q % 2 == 0 else _rev(natural, 16)), (q, lo, hi)
                seen[d] += 1
        assert np.all(seen == 1), q


def test_sr_probability_is_floor_of_p_times_2_16():
    # R10, pinned by counting: over the 2^16 draws, y rounds up exactly
    # floor(p * 2^16) times, p = (|y| - lo) / step computed exactly in rationals
    from fractions import Fraction
    rng = np.random.default_rng(3)
    ys = [0.0, 0.25, 0.3, 0.5, 0.74, 1.1, 1.999, 2.0, 2.5, 3.4, 3.999, 4.0, 5.0, 5.999, 6.0, 6.3, -0.3, -2.5]
    ys += [float(v) for v in rng.uniform(0, 6, 40).astype(np.float32)]
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for y in ys:
        y = float(np.float32(y))
        a = Fraction(abs(y))
        if a >= 6:
            want_up, lo = 0, Fraction(6)
        else:
            step = Fraction(1, 2) if a < 2 else (Fraction(1) if a < 4 else Fraction(2))
            lo = (a // step) * step
            want_up = int(((a - lo) / step) * 65536)        # floor
        codes = [O.e2m1_encode_sr(y, r) for r in range(1 << 16)]
        mags = [O.e2m1_decode(c & 7) for c in codes]
        ups = sum(1 for m in mags if m > lo)
        assert ups == want_up, (y, ups, want_up)
        assert all(m in (float(lo), float(min(lo + (step if a < 6 else 0), 6))) for m in mags) if a < 6 else \
            all(m == 6.0 for m in mags)
        # the draws that round up are the largest ones
        if 0 < ups < 65536:
            assert mags[65535 - ups] == float(lo) and mags[65536 - ups] > float(lo)


def test_sr_worked_example():
    # 3.4 between 3 and 4: P(4) = 0.4, P(3) = 0.6 (the page's worked example),
    # to within the draws' resolution of 2^-16
    (val, lo, hi, p_lo, p_hi), = [[float(t) for t in r] for r in _rows("sr_worked_example.txt")]
    n = 1 << 16
    ups = 0
    for r in range(n):
        v = O.e2m1_decode(O.e2m1_encode_sr(val, r))
        assert v in (lo, hi)
        ups += v == hi
    assert abs(ups / n - p_hi) < 2.0 / n
    assert abs((n - ups) / n - p_lo) < 2.0 / n


def test_sr_unbiased_over_draws():
    # A tensor whose amax is 2688 gives S_enc = 1; blocks whose max is 6 get
    # scale 1, so y = x and SR must average to x.
    C = 16 * 2048
    x = np.zeros((1, C), dtype=np.float32)
    x[0, 0::16] = 6.0
    x[0, 0] = 2688.0  # the tensor max, alone in block 0
    vals = np.float32([0.3, 1.1, 2.7, 3.40625, 5.0])
    for b in range(1, 2048):
        x[0, b * 16 + 1:(b + 1) * 16] = vals[b % len(vals)]
    xb = _bf16(x)
    codes, sf = O.quantize_row(xb, 2688.0, sr=True, seed=7)
    assert np.all(sf[0, 1:] == 0x38)  # scale exactly 1
    deq = np.array([O.e2m1_decode(c) for c in codes[0]])
    for k, v in enumerate(vals):
        v = float(_bf16([v]).float()[0])
        sel = [b * 16 + j for b in range(1, 2048) if b % len(vals) == k for j in range(1, 16)]
        m = deq[sel].mean()
        step = 0.5 if v < 2 else (1.0 if v < 4 else 2.0)
        sigma = step / 2                     # a Bernoulli step has std <= step / 2
        assert abs(m - v) <= 5 * sigma / math.sqrt(len(sel))


def test_sr_determinism_and_domains():
    x = synth.normal(64, 64, 11, std=1e-3)
    a = O.amax(x)
    c1, _ = O.quantize_row(x, a, sr=True, seed=5)
    c2, _ = O.quantize_row(x, a, sr=True, seed=5)
    c3, _ = O.quantize_row(x, a, sr=True, seed=6)
    assert np.array_equal(c1, c2) and not np.array_equal(c1, c3)
    # row and column domains draw independent words for the same element
    ct, _ = O.quantize_col(x, a, rht=False, sr=True, seed=5)
    assert not np.array_equal(ct.T, c1)


# ----------------------------------------------------------------- hadamard
def _hadamard16():
    i = np.arange(16)
    return np.array([[(-1) ** bin(a & b).count("1") for b in i] for a in i], dtype=np.float64)


def test_rht_is_quarter_h16_diag_signs():
    H = _hadamard16()
    assert np.array_equal(H @ H.T, 16 * np.eye(16))
    s = O.rht_signs()
    w = O.philox4x32_10([0, 0, 2, 0], [0, 0])[0]
    assert np.array_equal(s, np.where([(int(w) >> j) & 1 for j in range(16)], -1.0, 1.0).astype(np.float32))
    Q = np.stack([O.rht16_f32(np.eye(16, dtype=np.float32)[j]) for j in range(16)], axis=1)
    assert np.array_equal(Q, 0.25 * H * s[None, :])     # exact: one-hot columns


def test_rht_orthogonal_in_fp64():
    rng = np.random.default_rng(1)
    for _ in range(100):
        a, b = rng.standard_normal(16), rng.standard_normal(16)
        qa, qb = O.rht16_f64(a), O.rht16_f64(b)
        assert abs(qa @ qb - a @ b) <= 1e-12 * (np.abs(a) @ np.abs(b) + 1)
        assert abs(np.linalg.norm(qa) - np.linalg.norm(a)) <= 1e-12 * np.linalg.norm(a)


def test_rht_fp32_within_rounding_of_fp64():
    rng = np.random.default_rng(2)
    for _ in range(200):
        a = rng.standard_normal(16).astype(np.float32)
        y32 = O.rht16_f32(a).astype(np.float64)
        y64 = O.rht16_f64(a.astype(np.float64))
        # four levels of FP32 adds: relative error at most ~4 ulp of sum |a|
        assert np.all(np.abs(y32 - y64) <= 4 * 2.0 ** -24 * np.abs(a).sum() * 0.25 + 1e-30)


# ----------------------------------------------------------------- quantization
def test_global_scales():
    se, sg = O.global_scales(3.0)
    assert se == np.float32(2688.0) / np.float32(3.0) and sg == np.float32(3.0) / np.float32(2688.0)
    assert O.global_scales(0.0) == (1.0, 1.0)


def test_amax_closed_form():
    x = synth.normal(37, 48, 3)
    assert O.amax(x) == float(x.float().abs().max())
    assert O.amax(torch.zeros(4, 16, dtype=torch.bfloat16)) == 0.0


def test_amax_rht_matches_explicit_transform():
    x = synth.normal(64, 8, 4)
    xf = x.float().numpy()
    want = 0.0
    for tb in range(4):
        for c in range(8):
            want = max(want, float(np.abs(O.rht16_f32(xf[tb * 16:(tb + 1) * 16, c])).max()))
    assert O.amax_rht(x) == want


def _representable_tensor(R, C, rng):
    # blocks c_i * 2^k with max |c_i| = 6, 2^k in [2^-9, 2^8]; one element 2688
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    x = np.zeros((R, C))
    for r in range(R):
        for b in range(C // 16):
            k = rng.integers(-9, 9)
            c = grid[rng.integers(0, 8, 16)] * rng.choice([-1, 1], 16)
            c[rng.integers(0, 16)] = 6.0 * rng.choice([-1, 1])
            x[r, b * 16:(b + 1) * 16] = c * 2.0 ** k
    x[0, :16] = np.array([2688, 672, 0, -448, 224, 1344, -2688, 0, 448, 896, 1792, -224, 0, 0, -672, 0])
    return x


def test_row_quantize_round_trip_exact():
    rng = np.random.default_rng(3)
    x = _representable_tensor(8, 128, rng)
    xb = _bf16(x)
    assert np.array_equal(xb.float().numpy(), x)
    a = O.amax(xb)
    assert a == 2688.0
    codes, sf = O.quantize_row(xb, a)
    se, sg = O.global_scales(a)
    assert se == 1.0 and sg == 1.0
    assert np.array_equal(O.dequantize(codes, sf, sg), x)
    assert sf[0, 0] == 0x7E                       # the 2688 block takes scale 448


def test_col_without_rht_is_row_of_transpose():
    x = synth.activations(64, 96, 5)
    a = O.amax(x)
    ct, st = O.quantize_col(x, a)
    cr, sr_ = O.quantize_row(x.T.contiguous(), a)
    assert np.array_equal(ct, cr) and np.array_equal(st, sr_)


def test_col_rht_codes_within_rounding_of_transformed_values():
    x = synth.activations(64, 32, 6)
    a = O.amax_rht(x)
    codes, sf = O.quantize_col(x, a, rht=True)
    se, sg = O.global_scales(a)
    xf = x.float().numpy()
    for c in range(32):
        for tb in range(4):
            y = O.rht16_f32(xf[tb * 16:(tb + 1) * 16, c]).astype(np.float64)
            s_b = O.e4m3_decode(sf[c, tb])
            deq = np.array([O.e2m1_decode(q) for q in codes[c, tb * 16:(tb + 1) * 16]]) * s_b * sg
            # RN error of a scaled value: half a grid step (<= 1) times the block scale,
            # plus the saturation margin of an RN-rounded scale (<= 6/16 of a step)
            assert np.all(np.abs(deq - y) <= (1.0 + 0.375) * s_b * sg + 1e-6 * np.abs(y))


def test_2d_transpose_invariance():
    w = synth.weights(64, 96, 8, std=1.0)
    a = O.amax(w)
    c, t = O.quantize_2d(w, a)
    cT, tT = O.quantize_2d(w.T.contiguous(), a)
    assert np.array_equal(c, cT.T) and np.array_equal(t, tT.T)
    (rc, rs), (cc, cs) = O.expand_2d(c, t)
    assert np.array_equal(cc, cT) and np.array_equal(cs, np.repeat(tT, 16, axis=0))


def test_2d_equals_1d_when_tile_rows_share_block_max():
    # If every row of a 16x16 tile holds the tile's max, the 1x16 and 16x16
    # scales coincide and so do the codes.
    rng = np.random.default_rng(9)
    w = rng.standard_normal((32, 32)).astype(np.float32)
    w[:, 0] = 4.0
    w[:, 16] = -4.0
    wb = _bf16(w)
    a = O.amax(wb)
    c2, _ = O.quantize_2d(wb, a)
    c1, _ = O.quantize_row(wb, a)
    assert np.array_equal(c1, c2)


# ----------------------------------------------------------------- layouts
def test_scale_swizzle_is_a_bijection():
    for R, S in ((128, 4), (256, 16), (384, 12)):
        offs = sorted(O.sf_offset(r, c, S) for r in range(R) for c in range(S))
        assert offs == list(range(R * S))


def test_swizzle_padding_zero_and_pack_order():
    sf = np.arange(1, 1 + 130 * 5, dtype=np.uint32).reshape(130, 5) % 251 + 1
    out = O.swizzle_scales(sf.astype(np.uint8))
    assert out.size == 256 * 8 and np.count_nonzero(out) == 130 * 5
    codes = np.array([[1, 2, 15, 0]], dtype=np.uint8)
    assert list(O.pack_nibbles(codes)[0]) == [0x21, 0x0F]


# ----------------------------------------------------------------- gemm
def test_gemm_matches_numpy_on_dequantized_operands():
    x, w, _ = synth.workload_inputs("tiny")
    ax, aw = O.amax(x), O.amax(w)
    ca, sa = O.quantize_row(x, ax)
    cb, sb = O.quantize_row(w, aw)
    sga, sgb = O.global_scales(ax)[1], O.global_scales(aw)[1]
    D, S = O.gemm(ca, sa, sga, cb, sb, sgb)
    ref = O.dequantize(ca, sa, sga) @ O.dequantize(cb, sb, sgb).T
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-12)
    assert np.all(S >= np.abs(D) * (1 - 1e-12))
    pairs = np.array([[0, 0], [5, 77], [127, 127]])
    Ds, Ss = O.gemm(ca, sa, sga, cb, sb, sgb, pairs=pairs)
    assert np.array_equal(Ds, D[pairs[:, 0], pairs[:, 1]])


def test_gemm_integer_special_case_exact():
    rng = np.random.default_rng(4)
    M, N, K = 16, 24, 64
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cb = rng.integers(0, 16, (N, K)).astype(np.uint8)
    ones_a = np.full((M, K // 16), 0x38, np.uint8)
    ones_b = np.full((N, K // 16), 0x38, np.uint8)
    D, _ = O.gemm(ca, ones_a, 1.0, cb, ones_b, 1.0)
    val = {c: O.e2m1_decode(c) for c in range(16)}
    ia = np.vectorize(lambda c: int(round(2 * val[int(c)])))(ca).astype(np.int64)
    ib = np.vectorize(lambda c: int(round(2 * val[int(c)])))(cb).astype(np.int64)
    assert np.array_equal(D * 4, (ia @ ib.T).astype(np.float64))


def test_scale_offsets_match_documented_tile_layout():
    rows = _rows("sf_layout.txt")
    assert len(rows) >= 10
    for r, c, sp, off in ([int(t) for t in row] for row in rows):
        assert O.sf_offset(r, c, sp) == off, (r, c, sp)


# ----------------------------------------------------------------- row blocks of a larger tensor (R12)
@pytest.mark.parametrize("row0,rows", [(0, 32), (16, 48), (64, 16), (80, 48)])
def test_row_block_quantize_equals_slice_of_whole_tensor(row0, rows):
    # element (r, c) of a block that starts at row row0 draws the SR word of
    # element (row0 + r, c) of the whole tensor, so quantizing the block with
    # its row offset must reproduce the whole tensor's codes for those rows
    x = synth.gradients(128, 96, 31)
    a, ar = O.amax(x), O.amax_rht(x)
    blk = x[row0:row0 + rows].contiguous()
    whole_r = O.quantize_row(x, a, sr=True, seed=77)
    part_r = O.quantize_row(blk, a, sr=True, seed=77, row0=row0)
    assert np.array_equal(part_r[0], whole_r[0][row0:row0 + rows])
    assert np.array_equal(part_r[1], whole_r[1][row0:row0 + rows])
    whole_c = O.quantize_col(x, ar, rht=True, sr=True, seed=77)
    part_c = O.quantize_col(blk, ar, rht=True, sr=True, seed=77, row0=row0)
    assert np.array_equal(part_c[0], whole_c[0][:, row0:row0 + rows])
    assert np.array_equal(part_c[1], whole_c[1][:, row0 // 16:(row0 + rows) // 16])
    if row0:
        # the offset matters: without it the block draws other words
        assert not np.array_equal(O.quantize_row(blk, a, sr=True, seed=77)[0], part_r[0])


def test_row_offset_reaches_the_counter_high_word():
    # blocks whose counters g = (row0 + r) * C/16 + b pass 2^32: their draws are
    # those of the whole tensor's blocks, read one by one from the generator
    C, rows = 64, 16
    row0 = (1 << 36) // C - 8            # the rows straddle block counter 2^32
    x = synth.gradients(rows, C, 32)
    a = O.amax(x)
    codes, sf = O.quantize_row(x, a, sr=True, seed=5, row0=row0)
    S_enc = float(O.global_scales(a)[0])
    xf = x.float().numpy()
    crossed = False
    for r in (0, 7, 8, 15):
        for b in range(C // 16):
            g = (row0 + r) * (C // 16) + b
            crossed |= g >= 1 << 32
            draws = O.sr_block_draws(5, g, 0)
            blk = xf[r, b * 16:(b + 1) * 16]
            sb = O.e4m3_decode(sf[r, b])
            for i in range(16):
                y = np.float32(blk[i]) * (np.float32(S_enc) / np.float32(sb)) if sb else np.float32(0)
                want = O.e2m1_encode_sr(float(y), int(draws[i])) if sb else 0
                assert codes[r, b * 16 + i] == want, (r, b, i)
    assert crossed


def test_column_blocks_key_their_own_counters_past_2_32():
    # R11 for the column copy: the block of channel c and tokens 16tb.. of rows
    # row0.. of a larger tensor keys g = row0*C/16 + tb*C + c; here g passes
    # 2^32, and every code equals the rule applied to that block's draws
    C, rows = 64, 32
    row0 = (1 << 36) // C - 16           # a multiple of 16: blocks straddle counter 2^32
    x = synth.gradients(rows, C, 34)
    a = O.amax(x)
    codes_t, sf_t = O.quantize_col(x, a, sr=True, seed=9, row0=row0)
    S_enc = float(O.global_scales(a)[0])
    xf = x.float().numpy()
    crossed = below = False
    for c in (0, 1, 31, 63):
        for tb in range(rows // 16):
            g = (row0 * C) // 16 + tb * C + c
            crossed |= g >= 1 << 32
            below |= g < 1 << 32
            draws = O.sr_block_draws(9, g, 1)
            sb = O.e4m3_decode(sf_t[c, tb])
            for i in range(16):
                v = np.float32(xf[tb * 16 + i, c])
                y = v * (np.float32(S_enc) / np.float32(sb)) if sb else np.float32(0)
                want = O.e2m1_encode_sr(float(y), int(draws[i])) if sb else 0
                assert codes_t[c, tb * 16 + i] == want, (c, tb, i)
    assert crossed and below


# ----------------------------------------------------------------- non-finite inputs (R25)
def test_amax_propagates_nan_and_inf_like_numpy():
    x = synth.normal(48, 64, 33, std=2.0)
    for planted in (float("inf"), float("-inf"), float("nan")):
        y = x.clone()
        y[17, 9] = planted
        want = np.max(np.abs(y.float().numpy()))        # numpy's max propagates NaN
        got = O.amax(y)
        assert (math.isnan(got) and math.isnan(want)) or got == want, planted
        assert math.isnan(O.amax_rht(y)), planted
    assert O.amax(x) == np.max(np.abs(x.float().numpy()))


@pytest.mark.parametrize("amax", [float("inf"), float("nan")])
def test_nonfinite_amax_flags_every_copy(amax):
    x = synth.normal(32, 64, 34)
    for codes, sf in (O.quantize_row(x, amax), O.quantize_row(x, amax, sr=True, seed=3),
                      O.quantize_col(x, amax, rht=True, sr=True, seed=3), O.quantize_2d(x, amax)):
        assert not codes.any() and np.all(sf == 0x7F)
        assert math.isnan(O.e4m3_decode(0x7F))
    s_enc, s_g = O.global_scales(amax)
    assert not math.isfinite(s_g)
