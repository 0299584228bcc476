"""The C-ABI library loads, exports every declared symbol, and its host-only
logic (size queries, argument checks) behaves as declared.  CPU only: no call
here reaches a kernel."""
import ctypes
import os
import re

import pytest

import oracle as O
from nvfp4_bit_microscaled_b200 import _lib, build as libbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.PROTOTYPES, f"{n} has no ctypes prototype"


def test_size_queries(L):
    assert L.nvfp4_data_bytes(128, 256) == 128 * 128
    assert L.nvfp4_scale_bytes(128, 256) == 128 * 16
    assert L.nvfp4_scale_bytes(130, 80) == 256 * 8          # rows pad to 128, scale cols to 4
    assert L.nvfp4_data_bytes(0, 16) == 0
    ws = L.nvfp4_linear_workspace_bytes(128, 256, 128)
    assert ws >= 256 + 3 * (128 * 256 // 2) + 3 * (128 * 128 // 2)


def test_rht_signs_match_oracle(L):
    m = L.nvfp4_rht_sign_mask()
    s = O.rht_signs()
    assert [((m >> j) & 1) == 1 for j in range(16)] == [bool(v < 0) for v in s]


def test_status_strings(L):
    assert L.nvfp4_status_string(0) == b"ok"
    assert L.nvfp4_version() == 1
    for k in range(9):
        assert L.nvfp4_status_string(k)


def test_last_cuda_error_starts_clear(L):
    name = ctypes.c_char_p()
    assert L.nvfp4_last_cuda_error(None) == 0
    assert L.nvfp4_last_cuda_error(ctypes.byref(name)) == 0
    assert name.value == b"cudaSuccess"


def _t(rows, cols, data=4096, scales=8192, gs=16384):
    return _lib.Nvfp4Tensor(data, scales, gs, rows, cols)


def test_argument_checks_return_before_any_launch(L):
    fake = 1 << 20                              # never dereferenced: checks fail first
    st = L.nvfp4_amax(None, 4, 16, 16, 0, fake, None)
    assert st == 1
    assert L.nvfp4_amax(fake, 4, 16, 8, 0, fake, None) == 2          # ld < C
    assert L.nvfp4_amax(fake + 8, 4, 16, 16, 0, fake, None) == 3     # misaligned input
    assert L.nvfp4_amax(fake, 20, 16, 16, 1, fake, None) == 2        # RHT needs R % 16 == 0
    row = _t(16, 32)
    q = L.nvfp4_quantize
    assert q(fake, 16, 32, 32, 9, 0, 0, 0, fake, ctypes.byref(row), None, None) == 1   # bad mode
    assert q(fake, 16, 32, 32, _lib.ROW, 1, 0, 0, fake, ctypes.byref(row), None, None) == 4  # RHT on row copy
    assert q(fake, 16, 32, 32, _lib.TWO_D, 0, 1, 0, fake, ctypes.byref(row), None, None) == 4  # SR on weights
    assert q(fake, 16, 24, 24, _lib.ROW, 0, 0, 0, fake, ctypes.byref(_t(16, 24)), None, None) == 2  # C % 16
    assert q(fake, 16, 32, 32, _lib.ROW, 0, 0, 0, fake, ctypes.byref(_t(16, 64)), None, None) == 2  # desc shape
    assert q(fake, 16, 32, 32, _lib.ROW, 0, 0, 0, fake, None, None, None) == 1       # missing output
    assert q(fake, 16, 32, 32, _lib.ROW, 0, 0, 0, fake, ctypes.byref(_t(16, 32, data=4100)), None, None) == 3
    a, b = _t(128, 256), _t(128, 256)
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(_t(128, 128)), fake, 0, 128, None) == 2  # K mismatch
    assert L.nvfp4_gemm(ctypes.byref(_t(128, 80)), ctypes.byref(_t(128, 80)), fake, 0, 128, None) == 2  # K % 32
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), fake, 7, 128, None) == 1     # bad dtype
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), fake + 4, 0, 128, None) == 3  # misaligned D
    assert L.nvfp4_linear_fwd(fake, fake, 100, 64, 64, fake, fake, 1 << 30, None) == 2
    assert L.nvfp4_linear_fwd(fake, fake, 64, 64, 64, fake, fake, 16, None) == 7        # workspace too small
    assert L.nvfp4_linear_bwd(fake, 64, 64, 64, 0, fake, fake, None, 1 << 30, None) == 7


def test_mx_sizes_and_argument_checks(L):
    assert L.nvfp4_mx_scale_bytes(128, 256) == 128 * 8
    assert L.nvfp4_mx_scale_bytes(130, 96) == 256 * 4          # rows pad to 128, scale cols (3) to 4
    fake = 1 << 20
    q = L.nvfp4_mx_quantize
    assert q(fake, 16, 48, 48, ctypes.byref(_t(16, 48)), None) == 2          # C % 32
    assert q(fake, 16, 64, 64, ctypes.byref(_t(16, 32)), None) == 2          # descriptor shape
    assert q(fake + 8, 16, 64, 64, ctypes.byref(_t(16, 64)), None) == 3      # misaligned input
    assert q(fake, 16, 64, 64, None, None) == 1
    g = L.nvfp4_mx_gemm
    a, b = _t(256, 256), _t(256, 256)
    assert g(ctypes.byref(a), ctypes.byref(_t(200, 256)), fake, 0, 200, None) == 2   # N % 16
    assert g(ctypes.byref(a), ctypes.byref(b), fake, 0, 128, None) == 2              # ldd < N
    assert g(ctypes.byref(_t(256, 80)), ctypes.byref(_t(256, 80)), fake, 0, 256, None) == 2  # K % 32
    assert g(ctypes.byref(a), ctypes.byref(b), fake + 4, 0, 256, None) == 3        # misaligned D


def test_gemm_amax_argument_checks(L):
    fake = 1 << 20
    g = L.nvfp4_gemm_amax
    a, b = _t(256, 256), _t(256, 256)
    assert g(ctypes.byref(a), ctypes.byref(b), fake, 1, 256, None, None) == 1             # no amax pointer
    assert g(ctypes.byref(a), ctypes.byref(b), fake, 1, 256, fake + 2, None) == 3         # misaligned amax
    assert g(ctypes.byref(a), ctypes.byref(_t(200, 256)), fake, 1, 200, fake, None) == 2  # N % 16 (as nvfp4_gemm)
    assert g(ctypes.byref(a), ctypes.byref(b), fake + 4, 1, 256, fake, None) == 3         # misaligned D
    assert g(None, ctypes.byref(b), fake, 1, 256, fake, None) == 1


def test_quantize_rows_argument_checks(L):
    fake = 1 << 20
    q = L.nvfp4_quantize_rows
    row, col = _t(32, 64), _t(64, 32)
    assert q(fake, 32, 64, 64, _lib.ROW, 0, 1, 0, 8, fake, ctypes.byref(row), None, None) == 2     # row0 % 16
    assert q(fake, 32, 64, 64, _lib.ROW, 0, 1, 0, -16, fake, ctypes.byref(row), None, None) == 2   # row0 < 0
    assert q(fake, 32, 64, 64, _lib.COL, 1, 1, 0, 1 << 40, fake, None, ctypes.byref(col), None) == 2  # too far
    assert q(fake, 32, 64, 64, _lib.TWO_D, 0, 0, 0, 16, fake, ctypes.byref(row), ctypes.byref(col), None) == 4
    assert q(fake, 32, 64, 64, _lib.ROW, 1, 1, 0, 16, fake, ctypes.byref(row), None, None) == 4    # RHT on rows
    assert q(None, 32, 64, 64, _lib.ROW, 0, 1, 0, 16, fake, ctypes.byref(row), None, None) == 1
    wide = _t(32, 1 << 24)
    assert q(fake, 32, 1 << 24, 1 << 24, _lib.ROW, 0, 1, 0, 1 << 39, fake, ctypes.byref(wide), None, None) == 2  # index overflow


def test_valid_calls_without_a_gpu_fail_loudly(L):
    # every argument is valid, so the call gets as far as asking CUDA for the
    # device: on a machine without one it must return an error, never compute
    # on the host (there is no fallback path)
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: this checks the no-GPU behaviour")
    buf = ctypes.create_string_buffer((1 << 17) + 16)  # room for every operand below, D included
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    st = L.nvfp4_amax(base, 16, 32, 32, 0, base + 4096, None)
    assert st in (5, 6)                                    # NVFP4_ERR_DEVICE / NVFP4_ERR_CUDA
    q = L.nvfp4_quantize
    row = _lib.Nvfp4Tensor(base + 8192, base + 16384, base + 32768, 16, 32)
    assert q(base, 16, 32, 32, _lib.ROW, 0, 0, 0, base + 4096, ctypes.byref(row), None, None) in (5, 6)
    a = _lib.Nvfp4Tensor(base + 8192, base + 16384, base + 32768, 128, 64)
    assert L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(a), base + 65536, 0, 128, None) in (5, 6)
    with pytest.raises(_lib.Nvfp4Error):
        _lib.check("nvfp4_amax", L.nvfp4_amax(base, 16, 32, 32, 0, base + 4096, None))
