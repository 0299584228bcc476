"""Data-parallel NVFP4 linear layer: tokens sharded over the ranks of a
torch.distributed process group (NCCL on GPUs), the weight replicated.

A DP training step of Y = X W^T needs two exchanges beyond the single-GPU
path ("Pretraining Large Language Models with NVFP4", sections 2A and 2B):

- the per-tensor scale of X, Q.X, dY and Q.dY comes from the amax of the
  whole batch (two-level scaling), so each pass all-reduces (MAX) its local
  amaxes, two floats in one collective, before any quantize kernel runs;
- the partial FP32 weight gradients of the ranks are summed (all-reduce SUM);
  on NCCL it is issued as soon as the wgrad GEMM is done and overlaps the
  dgrad half of the backward pass.

On the GPU the layer also runs independent branches on a second stream: W's
amax and 2D copies beside X's amax and copies in the forward, and the dY row
copy (SR) beside the wgrad GEMM in the backward.

Stochastic rounding draws are keyed by the element's index in the whole
batch (nvfp4_quantize_rows with row0 = rank * T_local), so every rank's
quantized copies are the matching slices of a one-GPU quantization of the
whole batch, bit for bit, and Y and dX are the matching rows of the one-GPU
outputs.  Only dW differs from the one-GPU result, by the order of the final
FP32 sum.  W is replicated, so its amax needs no exchange.

Every computation runs in libnvfp4.so; this module only sequences the calls
and the collectives.
"""
import torch
import torch.distributed as dist

from . import api


class DataParallelLinear:
    """One linear layer's forward and backward on this rank's T_local tokens.

    The quantized operands live in buffers owned by the object (the same
    operands nvfp4_linear_fwd keeps in its workspace); forward() must run
    before backward() for the same batch.

    timer: optional callable timer(kind, fn) that runs fn() (one library call
    or one collective) and may record CUDA events around it; kinds name the
    kernel ("amax_both", "quant_row", "gemm_fprop", ...) or the collective
    ("allreduce_amax", "allreduce_dw").
    """

    def __init__(self, T_local, Cin, Cout, device, group=None, timer=None):
        if T_local % 16 or Cin % 16 or Cout % 16:
            raise ValueError("T_local, Cin and Cout must be multiples of 16")
        self.group = group
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.T, self.Cin, self.Cout = T_local, Cin, Cout
        self.row0 = self.rank * T_local
        self.timer = timer
        dev = torch.device(device)
        q = api.empty_qtensor
        self.x_row, self.x_col = q(T_local, Cin, dev), q(Cin, T_local, dev)
        self.w_row, self.w_col = q(Cout, Cin, dev), q(Cin, Cout, dev)
        self.dy_row, self.dy_col = q(T_local, Cout, dev), q(Cout, T_local, dev)
        self.amax_x = torch.zeros(2, dtype=torch.float32, device=dev)   # [max|X|, max|Q X|]
        self.amax_w = torch.zeros(1, dtype=torch.float32, device=dev)
        self.amax_dy = torch.zeros(2, dtype=torch.float32, device=dev)  # [max|dY|, max|Q dY|]

    def _do(self, kind, fn):
        return self.timer(kind, fn) if self.timer is not None else fn()

    def _side(self, device):
        """A second CUDA stream of this layer's (None off the GPU)."""
        if device.type != "cuda":
            return None
        if getattr(self, "_side_stream", None) is None:
            self._side_stream = torch.cuda.Stream(device)
        return self._side_stream

    def _branch(self, side, fn):
        """Run fn on the side stream after the work enqueued so far on the
        current stream; returns the event the current stream must wait for."""
        if side is None:
            fn()
            return None
        cur = torch.cuda.current_stream()
        start = torch.cuda.Event()
        start.record(cur)
        with torch.cuda.stream(side):
            side.wait_event(start)
            fn()
            done = torch.cuda.Event()
            done.record(side)
        return done

    def _all_reduce(self, t, op):
        if self.world == 1:
            return
        if t.is_cuda and dist.get_backend(self.group) == "gloo":
            # gloo reduces host memory: stage through it (NCCL reduces in place on the device)
            h = t.cpu()
            dist.all_reduce(h, op=op, group=self.group)
            t.copy_(h)
        else:
            dist.all_reduce(t, op=op, group=self.group)

    def forward(self, X, W, Y=None):
        """Y[T_local, Cout] = X W^T (BF16) for this rank's tokens."""
        assert X.shape == (self.T, self.Cin) and W.shape == (self.Cout, self.Cin)
        d = self._do
        # W's amax and 2D copies on the side stream while X's are made on this one
        w_done = self._branch(self._side(X.device), lambda: (
            d("amax", lambda: api.amax(W, out=self.amax_w)),
            d("quant_2d", lambda: api.quantize(W, api.TWO_D, self.amax_w, row_out=self.w_row, col_out=self.w_col))))
        d("amax_both", lambda: api.amax(X, rht=2, out=self.amax_x))
        if self.world > 1:
            d("allreduce_amax", lambda: self._all_reduce(self.amax_x, dist.ReduceOp.MAX))
        # X's row copy (fprop) and RHT column copy (wgrad) from one read of X
        d("quant_rowcol_rht", lambda: api.quantize(X, api.ROWCOL, self.amax_x, rht=True, row_out=self.x_row,
                                                   col_out=self.x_col, row0=self.row0))
        if w_done is not None:
            torch.cuda.current_stream().wait_event(w_done)
        return d("gemm_fprop", lambda: api.gemm(self.x_row, self.w_row, api.OUT_BF16, out=Y))

    def backward(self, dY, seed, dX=None, dW=None):
        """(dX[T_local, Cin] BF16, dW[Cout, Cin] FP32 summed over the ranks).

        The wgrad half runs first, so that on NCCL the all-reduce of dW runs on
        the communicator's stream while the dY row copy and the dgrad GEMM
        compute; the call returns once both are done (stream order)."""
        assert dY.shape == (self.T, self.Cout)
        d = self._do
        d("amax_both", lambda: api.amax(dY, rht=2, out=self.amax_dy))
        if self.world > 1:
            d("allreduce_amax", lambda: self._all_reduce(self.amax_dy, dist.ReduceOp.MAX))
        d("quant_col_rht_sr", lambda: api.quantize(dY, api.COL, self.amax_dy[1:2], rht=True, sr=True, seed=seed,
                                                   col_out=self.dy_col, row0=self.row0))
        side = self._side(dY.device)
        start = None
        if side is not None:
            start = torch.cuda.Event()
            start.record(torch.cuda.current_stream())
        dW = d("gemm_wgrad", lambda: api.gemm(self.dy_col, self.x_col, api.OUT_F32, out=dW))
        # the dY row copy (SR) on the side stream, next to the wgrad GEMM: the
        # quantizer is bound by the integer ALU pipe, the GEMM by the tensor pipe.
        # Enqueued before the dW all-reduce, so that a host-staged (gloo) reduce
        # does not hold it back.
        row_sr = lambda: d("quant_row_sr", lambda: api.quantize(dY, api.ROW, self.amax_dy[0:1], sr=True, seed=seed,
                                                                row_out=self.dy_row, row0=self.row0))
        done = None
        if side is None:
            row_sr()
        else:
            with torch.cuda.stream(side):
                side.wait_event(start)
                row_sr()
                done = torch.cuda.Event()
                done.record(side)
        pending = None
        if self.world > 1:
            if dist.get_backend(self.group) == "nccl":
                pending = dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=self.group, async_op=True)
            else:
                d("allreduce_dw", lambda: self._all_reduce(dW, dist.ReduceOp.SUM))
        if done is not None:
            torch.cuda.current_stream().wait_event(done)
        dX = d("gemm_dgrad", lambda: api.gemm(self.dy_row, self.w_col, api.OUT_BF16, out=dX))
        if pending is not None:
            d("allreduce_dw_wait", pending.wait)   # the current stream waits for the all-reduce
        return dX, dW
