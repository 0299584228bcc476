"""Thin PyTorch-facing binding over the C ABI.

PyTorch provides device memory and the current CUDA stream; every step of the
computation runs in the library's sm_100a kernels.  Functions keep the C
names without the ``nvfp4_`` prefix.
"""
import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import COL, OUT_BF16, OUT_F32, ROW, ROWCOL, TWO_D, Nvfp4Tensor, check, lib

__all__ = ["QTensor", "empty_qtensor", "amax", "quantize", "copy_is_flagged", "gemm", "LinearWorkspace", "linear_fwd",
           "linear_bwd", "read_device_error", "wait_probe", "rht_sign_mask", "data_bytes", "scale_bytes",
           "ROW", "COL", "ROWCOL", "TWO_D", "OUT_F32", "OUT_BF16"]


def _stream(device=None):
    return torch.cuda.current_stream(device).cuda_stream


def data_bytes(rows, cols):
    return lib().nvfp4_data_bytes(rows, cols)


def scale_bytes(rows, cols):
    return lib().nvfp4_scale_bytes(rows, cols)


def rht_sign_mask():
    return lib().nvfp4_rht_sign_mask()


@dataclass
class QTensor:
    """A quantized K-major operand: packed codes, swizzled scales, decode scale."""
    data: torch.Tensor          # uint8 [rows, cols/2]
    scales: torch.Tensor        # uint8 [scale_bytes(rows, cols)]
    global_scale: torch.Tensor  # float32 [1]
    rows: int
    cols: int

    def desc(self):
        return Nvfp4Tensor(self.data.data_ptr(), self.scales.data_ptr(), self.global_scale.data_ptr(),
                           self.rows, self.cols)


def empty_qtensor(rows, cols, device):
    return QTensor(torch.empty(rows, cols // 2, dtype=torch.uint8, device=device),
                   torch.empty(scale_bytes(rows, cols), dtype=torch.uint8, device=device),
                   torch.empty(1, dtype=torch.float32, device=device), rows, cols)


def amax(x, rht=False, out=None):
    """max|x| (rht=0), max|Q x| along rows (rht=1), or both from one pass
    (rht=2: out[0] = max|x|, out[1] = max|Q x|) of a BF16 [R, C] tensor."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    if out is None:
        out = torch.empty(2 if int(rht) == 2 else 1, dtype=torch.float32, device=x.device)
    check("nvfp4_amax", lib().nvfp4_amax(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), int(rht),
                                         out.data_ptr(), _stream(x.device)))
    return out


def quantize(x, mode, amax_dev, rht=False, sr=False, seed=0, row_out=None, col_out=None, row0=0):
    """BF16 [R, C] -> (row copy, column copy); a copy the mode does not make is None.

    In TWO_D mode both copies are made unless row_out or col_out is False.
    ROWCOL with rht: the row copy is scaled by amax_dev[0] and the RHT column
    copy by amax_dev[1] (the two floats amax(x, rht=2) returns).
    row0 != 0 (nvfp4_quantize_rows): x is rows row0 .. of a larger tensor, and
    the SR draws are those of the whole tensor's elements.
    """
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    R, C = x.shape
    if mode == ROWCOL and rht:
        assert amax_dev.numel() >= 2, "ROWCOL with rht takes [amax of x, amax of Q x]"
    want_row = mode in (ROW, ROWCOL) or (mode == TWO_D and row_out is not False)
    want_col = mode in (COL, ROWCOL) or (mode == TWO_D and col_out is not False)
    if want_row and not isinstance(row_out, QTensor):
        row_out = empty_qtensor(R, C, x.device)
    if want_col and not isinstance(col_out, QTensor):
        col_out = empty_qtensor(C, R, x.device)
    rd = row_out.desc() if want_row else None
    cd = col_out.desc() if want_col else None
    if row0:
        st = lib().nvfp4_quantize_rows(x.data_ptr(), R, C, x.stride(0), mode, int(rht), int(sr), int(seed),
                                       int(row0), amax_dev.data_ptr(), ctypes.byref(rd) if rd else None,
                                       ctypes.byref(cd) if cd else None, _stream(x.device))
        check("nvfp4_quantize_rows", st)
    else:
        st = lib().nvfp4_quantize(x.data_ptr(), R, C, x.stride(0), mode, int(rht), int(sr), int(seed),
                                  amax_dev.data_ptr(), ctypes.byref(rd) if rd else None,
                                  ctypes.byref(cd) if cd else None, _stream(x.device))
        check("nvfp4_quantize", st)
    return (row_out if want_row else None), (col_out if want_col else None)


def copy_is_flagged(q):
    """Host-side check of a quantized copy: True when its per-tensor amax was
    not finite (a NaN or an infinity in the tensor), in which case the kernels
    wrote 0x7F (the E4M3 NaN) to every block scale, 0 to every code, and a
    non-finite decode scale.  Reads one float back (synchronizes the stream)."""
    return not torch.isfinite(q.global_scale).all().item()


def gemm(A, B, out_dtype=OUT_F32, out=None):
    """D[M, N] = s_gA s_gB sum_k A[m, k] B[n, k] (FP32 accumulation)."""
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(A.rows, B.rows, dtype=dt, device=A.data.device)
    ad, bd = A.desc(), B.desc()
    check("nvfp4_gemm", lib().nvfp4_gemm(ctypes.byref(ad), ctypes.byref(bd), out.data_ptr(), out_dtype,
                                         out.stride(0), _stream(out.device)))
    return out


def gemm_amax(A, B, out_dtype=OUT_BF16, out=None, amax_out=None):
    """gemm() that also returns max|D| over the stored outputs (a 1-float
    device tensor), reduced in the GEMM's epilogue: (D, amax)."""
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(A.rows, B.rows, dtype=dt, device=A.data.device)
    if amax_out is None:
        amax_out = torch.empty(1, dtype=torch.float32, device=out.device)
    ad, bd = A.desc(), B.desc()
    check("nvfp4_gemm_amax", lib().nvfp4_gemm_amax(ctypes.byref(ad), ctypes.byref(bd), out.data_ptr(), out_dtype,
                                                   out.stride(0), amax_out.data_ptr(), _stream(out.device)))
    return out, amax_out


# ---------------------------------------------------------------- MXFP4 comparison format
def mx_scale_bytes(rows, cols):
    return lib().nvfp4_mx_scale_bytes(rows, cols)


def mx_quantize(x, out=None):
    """BF16 [R, C] -> MXFP4 QTensor (1x32 blocks along C, UE8M0 scales, global_scale = 1)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    R, C = x.shape
    if out is None:
        out = QTensor(torch.empty(R, C // 2, dtype=torch.uint8, device=x.device),
                      torch.empty(mx_scale_bytes(R, C), dtype=torch.uint8, device=x.device),
                      torch.empty(1, dtype=torch.float32, device=x.device), R, C)
    d = out.desc()
    check("nvfp4_mx_quantize", lib().nvfp4_mx_quantize(x.data_ptr(), R, C, x.stride(0), ctypes.byref(d),
                                                       _stream(x.device)))
    return out


def mx_gemm(A, B, out_dtype=OUT_F32, out=None):
    """D[M, N] = sum_k A[m, k] B[n, k] on MXFP4 operands (FP32 accumulation)."""
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(A.rows, B.rows, dtype=dt, device=A.data.device)
    ad, bd = A.desc(), B.desc()
    check("nvfp4_mx_gemm", lib().nvfp4_mx_gemm(ctypes.byref(ad), ctypes.byref(bd), out.data_ptr(), out_dtype,
                                               out.stride(0), _stream(out.device)))
    return out


class LinearWorkspace:
    """Caller-owned workspace of the linear layer (quantized operands + scalars)."""

    WHICH = {"x_row": 0, "w_row": 1, "w_col": 2, "x_col": 3, "dy_row": 4, "dy_col": 5}

    def __init__(self, T, Cin, Cout, device):
        self.T, self.Cin, self.Cout = T, Cin, Cout
        self.nbytes = lib().nvfp4_linear_workspace_bytes(T, Cin, Cout)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)

    def tensor(self, name):
        """Descriptor of one quantized operand inside the workspace, as a QTensor view."""
        d = Nvfp4Tensor()
        check("nvfp4_linear_workspace_tensor",
              lib().nvfp4_linear_workspace_tensor(self.buf.data_ptr(), self.T, self.Cin, self.Cout,
                                                  self.WHICH[name], ctypes.byref(d)))
        base = self.buf.data_ptr()
        dv = self.buf[d.data - base:d.data - base + d.rows * d.cols // 2].view(d.rows, d.cols // 2)
        sb = scale_bytes(d.rows, d.cols)
        sv = self.buf[d.scales - base:d.scales - base + sb]
        gv = self.buf[d.global_scale - base:d.global_scale - base + 4].view(torch.float32)
        return QTensor(dv, sv, gv, d.rows, d.cols)


def linear_fwd(X, W, ws, Y=None):
    T, Cin = X.shape
    Cout = W.shape[0]
    if Y is None:
        Y = torch.empty(T, Cout, dtype=torch.bfloat16, device=X.device)
    check("nvfp4_linear_fwd", lib().nvfp4_linear_fwd(X.data_ptr(), W.data_ptr(), T, Cin, Cout, Y.data_ptr(),
                                                     ws.buf.data_ptr(), ws.nbytes, _stream(X.device)))
    return Y


def linear_bwd(dY, ws, seed, dX=None, dW=None):
    T, Cout = dY.shape
    Cin = ws.Cin
    if dX is None:
        dX = torch.empty(T, Cin, dtype=torch.bfloat16, device=dY.device)
    if dW is None:
        dW = torch.empty(Cout, Cin, dtype=torch.float32, device=dY.device)
    check("nvfp4_linear_bwd", lib().nvfp4_linear_bwd(dY.data_ptr(), T, Cin, Cout, int(seed), dX.data_ptr(),
                                                     dW.data_ptr(), ws.buf.data_ptr(), ws.nbytes,
                                                     _stream(dY.device)))
    return dX, dW


def read_device_error(clear=True):
    v = ctypes.c_uint(0)
    check("nvfp4_read_device_error", lib().nvfp4_read_device_error(ctypes.byref(v), int(clear)))
    return v.value


def wait_probe(timeout_us, device=None):
    check("nvfp4_wait_probe", lib().nvfp4_wait_probe(int(timeout_us), _stream(device)))


def selftest_scale_division():
    """(bad_quotients, bad_codes) of the kernels' divide-by-6 against IEEE division on every
    non-negative finite float; both are 0 on a correct build."""
    q, c = ctypes.c_uint64(0), ctypes.c_uint64(0)
    check("nvfp4_selftest_scale_division",
          lib().nvfp4_selftest_scale_division(ctypes.byref(q), ctypes.byref(c)))
    return q.value, c.value


def selftest_sr_rounding():
    """(mismatches, checked) of the stochastic-rounding conversion against its rule,
    every 16-bit draw of every lane for 8192 values; mismatches is 0 on a correct build."""
    m, c = ctypes.c_uint64(0), ctypes.c_uint64(0)
    check("nvfp4_selftest_sr_rounding", lib().nvfp4_selftest_sr_rounding(ctypes.byref(m), ctypes.byref(c)))
    return m.value, c.value


# ---------------------------------------------------------------- layer precision policy
def block_uses_bf16(block, n_blocks, first=2, last=8):
    """Whether transformer block `block` (0-based, of n_blocks) keeps its linear
    layers in BF16 instead of NVFP4.  "Pretraining Large Language Models with
    NVFP4", section 2B.1: the most sensitive layers, mainly the last ones, stay
    in high precision; the 12B run kept the first two and the last eight blocks
    in BF16 (about 16% of the linear layers).  A host-side switch: the BF16
    layers are the framework's own and do not go through this library."""
    if not 0 <= block < n_blocks:
        raise ValueError(f"block {block} outside 0..{n_blocks - 1}")
    return block < first or block >= n_blocks - last
