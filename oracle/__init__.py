"""CPU oracle for the NVFP4 quantized linear layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it, and it never imports the product.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, FP32 steps in source order,
FP64 GEMM); this module only marshals numpy arrays through ctypes.  The readings
R1..R18 (NVFP4) and R21..R24 (the MXFP4 comparison format) that fix what the
pages leave open are listed at the top of that file.

Non-finite inputs follow reading R25 (NaN-propagating amax; a copy whose amax
is not finite has all scales 0x7F, all codes 0).

Parity unpinned: the storage layouts (R17 nibble order, R18 scale swizzle),
the op-order readings (R4, R6, R9, R16) and the MXFP4 scale rule and clipping
(R23, R24: the OCP Microscaling definition the pages name but do not spell
out) have no pin in the pages; everything else is pinned by
``tests/test_oracle_pins.py`` and ``tests/test_oracle_mx_pins.py``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        sig = {
            "orc_e2m1_decode": (ctypes.c_double, [ctypes.c_int]),
            "orc_e4m3_decode": (ctypes.c_double, [ctypes.c_int]),
            "orc_e2m1_encode_rn": (ctypes.c_int, [ctypes.c_float]),
            "orc_e4m3_encode_rn_sat": (ctypes.c_int, [ctypes.c_float]),
            "orc_e2m1_encode_sr": (ctypes.c_int, [ctypes.c_float, ctypes.c_uint32]),
            "orc_philox4x32_10": (None, [_u32p, _u32p, _u32p]),
            "orc_sr_block_words": (None, [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32, _u32p]),
            "orc_sr_draw16": (ctypes.c_uint32, [ctypes.c_uint32, ctypes.c_int]),
            "orc_sr_block_draws": (None, [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32, _u32p]),
            "orc_rht_signs": (None, [_f32p]),
            "orc_rht16_f32": (None, [_f32p, _f32p]),
            "orc_rht16_f64": (None, [_f64p, _f64p]),
            "orc_amax": (ctypes.c_float, [_u16p, _i64, _i64, _i64]),
            "orc_amax_rht": (ctypes.c_float, [_u16p, _i64, _i64, _i64]),
            "orc_global_scales": (None, [ctypes.c_float, _f32p]),
            "orc_quantize_row": (None, [_u16p, _i64, _i64, _i64, ctypes.c_float, ctypes.c_int,
                                        ctypes.c_uint64, _i64, _u8p, _u8p]),
            "orc_quantize_col": (None, [_u16p, _i64, _i64, _i64, ctypes.c_float, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_uint64, _i64, _u8p, _u8p]),
            "orc_quantize_2d": (None, [_u16p, _i64, _i64, _i64, ctypes.c_float, _u8p, _u8p]),
            "orc_pack_nibbles": (None, [_u8p, _i64, _i64, _u8p]),
            "orc_sf_offset": (_i64, [_i64, _i64, _i64]),
            "orc_swizzle_scales": (None, [_u8p, _i64, _i64, _u8p]),
            "orc_gemm": (None, [_u8p, _u8p, ctypes.c_float, _u8p, _u8p, ctypes.c_float, _i64, _i64,
                                _i64, _i64p, _i64, _f64p, _f64p]),
            "orc_dequantize": (None, [_u8p, _u8p, ctypes.c_float, _i64, _i64, _f64p]),
            "orc_e8m0_decode": (ctypes.c_double, [ctypes.c_int]),
            "orc_mx_scale_exponent": (ctypes.c_int, [ctypes.c_float]),
            "orc_mx_quantize_row": (None, [_u16p, _i64, _i64, _i64, _u8p, _u8p]),
            "orc_mx_gemm": (None, [_u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i64p, _i64, _f64p, _f64p]),
            "orc_num_threads": (ctypes.c_int, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _p(a, t):
    return a.ctypes.data_as(t)


def _bf16_bits(x):
    """Accept a numpy uint16 array of BF16 bit patterns or a torch bfloat16 tensor."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(getattr(x, "dtype", "")) == "torch.bfloat16":
        import torch
        x = x.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16 and x.ndim == 2
    return x


# ---------------------------------------------------------------- formats
def e2m1_decode(code):
    return lib().orc_e2m1_decode(int(code))


def e4m3_decode(b):
    return lib().orc_e4m3_decode(int(b))


def e2m1_encode_rn(y):
    return lib().orc_e2m1_encode_rn(float(y))


def e4m3_encode_rn_sat(d):
    return lib().orc_e4m3_encode_rn_sat(float(d))


def e2m1_encode_sr(y, r16):
    """Stochastic rounding of y with the 16-bit draw r16 (R10)."""
    return lib().orc_e2m1_encode_sr(float(y), int(r16) & 0xFFFF)


# ---------------------------------------------------------------- philox / rht
def philox4x32_10(ctr, key):
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(_p(c, _u32p), _p(k, _u32p), _p(out, _u32p))
    return out


def sr_block_words(seed, g, domain):
    """The four Philox words of the block keyed g (R11)."""
    out = np.zeros(4, dtype=np.uint32)
    lib().orc_sr_block_words(int(seed), int(g), int(domain), _p(out, _u32p))
    return out


def sr_draw16(word, q):
    """The 16-bit draw of element q (0..3) of a word (R10)."""
    return lib().orc_sr_draw16(int(word) & 0xFFFFFFFF, int(q))


def sr_block_draws(seed, g, domain):
    """The 16-bit draws of the sixteen elements of the block keyed g."""
    out = np.zeros(16, dtype=np.uint32)
    lib().orc_sr_block_draws(int(seed), int(g), int(domain), _p(out, _u32p))
    return out


def rht_signs():
    s = np.zeros(16, dtype=np.float32)
    lib().orc_rht_signs(_p(s, _f32p))
    return s


def rht16_f32(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.zeros(16, dtype=np.float32)
    lib().orc_rht16_f32(_p(x, _f32p), _p(y, _f32p))
    return y


def rht16_f64(x):
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(16, dtype=np.float64)
    lib().orc_rht16_f64(_p(x, _f64p), _p(y, _f64p))
    return y


# ---------------------------------------------------------------- tensors
def amax(x):
    x = _bf16_bits(x)
    return lib().orc_amax(_p(x, _u16p), x.shape[0], x.shape[1], x.shape[1])


def amax_rht(x):
    x = _bf16_bits(x)
    assert x.shape[0] % 16 == 0
    return lib().orc_amax_rht(_p(x, _u16p), x.shape[0], x.shape[1], x.shape[1])


def global_scales(a):
    """Returns (S_enc, s_g) as numpy float32 scalars."""
    out = np.zeros(2, dtype=np.float32)
    lib().orc_global_scales(float(a), _p(out, _f32p))
    return out[0], out[1]


def quantize_row(x, a, sr=False, seed=0, row0=0):
    """Row-wise 1x16.  Returns (codes [R, C] u8, sf [R, C/16] u8).  row0: x is
    rows row0.. of a larger tensor with C columns, whose element indices key the
    SR draws (R12)."""
    x = _bf16_bits(x)
    R, C = x.shape
    codes = np.zeros((R, C), dtype=np.uint8)
    sf = np.zeros((R, C // 16), dtype=np.uint8)
    lib().orc_quantize_row(_p(x, _u16p), R, C, C, float(a), int(bool(sr)), int(seed), int(row0) * C,
                           _p(codes, _u8p), _p(sf, _u8p))
    return codes, sf


def quantize_col(x, a, rht=False, sr=False, seed=0, row0=0):
    """Column-wise 1x16 along rows; transposed output (codes [C, R], sf [C, R/16]).
    row0 as in quantize_row."""
    x = _bf16_bits(x)
    R, C = x.shape
    codes = np.zeros((C, R), dtype=np.uint8)
    sf = np.zeros((C, R // 16), dtype=np.uint8)
    lib().orc_quantize_col(_p(x, _u16p), R, C, C, float(a), int(bool(rht)), int(bool(sr)), int(seed),
                           int(row0) * C, _p(codes, _u8p), _p(sf, _u8p))
    return codes, sf


def quantize_2d(w, a):
    """16x16 2D.  Returns (codes [N, K], sf_tile [N/16, K/16])."""
    w = _bf16_bits(w)
    N, K = w.shape
    codes = np.zeros((N, K), dtype=np.uint8)
    sft = np.zeros((N // 16, K // 16), dtype=np.uint8)
    lib().orc_quantize_2d(_p(w, _u16p), N, K, K, float(a), _p(codes, _u8p), _p(sft, _u8p))
    return codes, sft


def expand_2d(codes, sft):
    """Row copy and column copy of a 2D-quantized weight, each as (codes, sf)."""
    row_sf = np.repeat(sft, 16, axis=0)                 # [N, K/16]
    col_codes = np.ascontiguousarray(codes.T)           # [K, N]
    col_sf = np.ascontiguousarray(np.repeat(sft.T, 16, axis=0))  # [K, N/16]
    return (codes, np.ascontiguousarray(row_sf)), (col_codes, col_sf)


def pack_nibbles(codes):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    R, C = codes.shape
    out = np.zeros((R, C // 2), dtype=np.uint8)
    lib().orc_pack_nibbles(_p(codes, _u8p), R, C, _p(out, _u8p))
    return out


def sf_offset(r, c, Sp):
    return lib().orc_sf_offset(int(r), int(c), int(Sp))


def swizzle_scales(sf):
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    R, S = sf.shape
    Rp, Sp = (R + 127) // 128 * 128, (S + 3) // 4 * 4
    out = np.zeros(Rp * Sp, dtype=np.uint8)
    lib().orc_swizzle_scales(_p(sf, _u8p), R, S, _p(out, _u8p))
    return out


def gemm(ca, sa, sga, cb, sb, sgb, pairs=None):
    """FP64 D = dq(A) dq(B)^T.  Full [M, N] or sampled entries.  Returns (D, absum)."""
    ca, sa, cb, sb = (np.ascontiguousarray(t, dtype=np.uint8) for t in (ca, sa, cb, sb))
    M, K = ca.shape
    N = cb.shape[0]
    assert cb.shape[1] == K and sa.shape == (M, K // 16) and sb.shape == (N, K // 16)
    if pairs is None:
        D = np.zeros((M, N), dtype=np.float64)
        S = np.zeros((M, N), dtype=np.float64)
        lib().orc_gemm(_p(ca, _u8p), _p(sa, _u8p), float(sga), _p(cb, _u8p), _p(sb, _u8p), float(sgb),
                       M, N, K, None, 0, _p(D, _f64p), _p(S, _f64p))
    else:
        pr = np.ascontiguousarray(pairs, dtype=np.int64)
        n = pr.shape[0]
        D = np.zeros(n, dtype=np.float64)
        S = np.zeros(n, dtype=np.float64)
        lib().orc_gemm(_p(ca, _u8p), _p(sa, _u8p), float(sga), _p(cb, _u8p), _p(sb, _u8p), float(sgb),
                       M, N, K, _p(pr, _i64p), n, _p(D, _f64p), _p(S, _f64p))
    return D, S


def dequantize(codes, sf, sg):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    R, C = codes.shape
    out = np.zeros((R, C), dtype=np.float64)
    lib().orc_dequantize(_p(codes, _u8p), _p(sf, _u8p), float(sg), R, C, _p(out, _f64p))
    return out


# ---------------------------------------------------------------- MXFP4 (R21-R24)
def e8m0_decode(byte):
    return lib().orc_e8m0_decode(int(byte))


def mx_scale_exponent(bamax):
    return lib().orc_mx_scale_exponent(float(bamax))


def mx_quantize_row(x):
    """Row-wise 1x32 MXFP4.  Returns (codes [R, C] u8, sf [R, C/32] UE8M0 bytes)."""
    x = _bf16_bits(x)
    R, C = x.shape
    codes = np.zeros((R, C), dtype=np.uint8)
    sf = np.zeros((R, C // 32), dtype=np.uint8)
    lib().orc_mx_quantize_row(_p(x, _u16p), R, C, C, _p(codes, _u8p), _p(sf, _u8p))
    return codes, sf


def mx_dequantize(codes, sf):
    """FP64 values of an unpacked MXFP4 operand (codes [R, C], sf [R, C/32])."""
    grid = np.array([lib().orc_e2m1_decode(c) for c in range(16)])
    scale = np.array([lib().orc_e8m0_decode(b) for b in range(256)])
    return grid[codes] * np.repeat(scale[sf], 32, axis=1)


def mx_gemm(ca, sa, cb, sb, pairs=None):
    """FP64 D = dq(A) dq(B)^T on MXFP4 operands.  Full [M, N] or sampled entries.  Returns (D, absum)."""
    ca, sa, cb, sb = (np.ascontiguousarray(t, dtype=np.uint8) for t in (ca, sa, cb, sb))
    M, K = ca.shape
    N = cb.shape[0]
    assert cb.shape[1] == K and sa.shape == (M, K // 32) and sb.shape == (N, K // 32)
    pr = None if pairs is None else np.ascontiguousarray(pairs, dtype=np.int64)
    n = M * N if pr is None else pr.shape[0]
    D = np.zeros(n, dtype=np.float64)
    S = np.zeros(n, dtype=np.float64)
    lib().orc_mx_gemm(_p(ca, _u8p), _p(sa, _u8p), _p(cb, _u8p), _p(sb, _u8p), M, N, K,
                      None if pr is None else _p(pr, _i64p), 0 if pr is None else n, _p(D, _f64p), _p(S, _f64p))
    if pr is None:
        D, S = D.reshape(M, N), S.reshape(M, N)
    return D, S


def num_threads():
    return lib().orc_num_threads()


__all__ = [n for n in dir() if not n.startswith("_")]
