"""ctypes loader for libnvfp4.so (the C ABI declared in include/nvfp4.h).

Argument marshalling only.  There is no fallback: if the shared library is
missing or does not load, every call raises.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

NVFP4_OK = 0
NVFP4_ERR_CUDA = 6
STATUS_NAMES = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_SHAPE", 3: "NVFP4_ERR_ALIGN",
    4: "NVFP4_ERR_UNSUPPORTED", 5: "NVFP4_ERR_DEVICE", 6: "NVFP4_ERR_CUDA", 7: "NVFP4_ERR_WORKSPACE",
    8: "NVFP4_ERR_TIMEOUT",
}
ROW, COL, ROWCOL, TWO_D = 1, 2, 3, 4
OUT_F32, OUT_BF16 = 0, 1


class Nvfp4Tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class Nvfp4Error(RuntimeError):
    def __init__(self, fn, status, cuda_error=None):
        self.status = status
        self.cuda_error = cuda_error
        extra = f" ({cuda_error[1]}, code {cuda_error[0]})" if cuda_error else ""
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}{extra}")


_c = ctypes
_vp, _i64, _u64, _int, _u32 = _c.c_void_p, _c.c_int64, _c.c_uint64, _c.c_int, _c.c_uint32
_tp = _c.POINTER(Nvfp4Tensor)

PROTOTYPES = {
    "nvfp4_data_bytes": (_c.c_size_t, [_i64, _i64]),
    "nvfp4_scale_bytes": (_c.c_size_t, [_i64, _i64]),
    "nvfp4_amax": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _vp]),
    "nvfp4_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _u64, _vp, _tp, _tp, _vp]),
    "nvfp4_quantize_rows": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _u64, _i64, _vp, _tp, _tp, _vp]),
    "nvfp4_gemm": (_int, [_tp, _tp, _vp, _int, _i64, _vp]),
    "nvfp4_gemm_amax": (_int, [_tp, _tp, _vp, _int, _i64, _vp, _vp]),
    "nvfp4_linear_workspace_bytes": (_c.c_size_t, [_i64, _i64, _i64]),
    "nvfp4_linear_fwd": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _c.c_size_t, _vp]),
    "nvfp4_linear_bwd": (_int, [_vp, _i64, _i64, _i64, _u64, _vp, _vp, _vp, _c.c_size_t, _vp]),
    "nvfp4_linear_workspace_tensor": (_int, [_vp, _i64, _i64, _i64, _int, _tp]),
    "nvfp4_linear_fwd_noalloc": (_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "nvfp4_read_device_error": (_int, [_c.POINTER(_c.c_uint), _int]),
    "nvfp4_wait_probe": (_int, [_u32, _vp]),
    "nvfp4_rht_sign_mask": (_u32, []),
    "nvfp4_status_string": (_c.c_char_p, [_int]),
    "nvfp4_version": (_int, []),
    "nvfp4_last_cuda_error": (_int, [_c.POINTER(_c.c_char_p)]),
    "nvfp4_mx_scale_bytes": (_c.c_size_t, [_i64, _i64]),
    "nvfp4_mx_quantize": (_int, [_vp, _i64, _i64, _i64, _tp, _vp]),
    "nvfp4_mx_gemm": (_int, [_tp, _tp, _vp, _int, _i64, _vp]),
    "nvfp4_selftest_scale_division": (_int, [_c.POINTER(_c.c_uint64), _c.POINTER(_c.c_uint64)]),
    "nvfp4_selftest_sr_rounding": (_int, [_c.POINTER(_c.c_uint64), _c.POINTER(_c.c_uint64)]),
}

_LIB = None


def lib():
    """Load libnvfp4.so once; raise loudly if it is not there."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m nvfp4_bit_microscaled_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def check(fn_name, status):
    if status != NVFP4_OK:
        cuda_error = None
        if status == NVFP4_ERR_CUDA and _LIB is not None:
            name = _c.c_char_p()
            code = _LIB.nvfp4_last_cuda_error(_c.byref(name))
            cuda_error = (code, (name.value or b"?").decode())
        raise Nvfp4Error(fn_name, status, cuda_error)
