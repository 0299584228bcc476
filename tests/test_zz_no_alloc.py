"""nvfp4_linear_fwd_noalloc: the linear forward for callers that cannot allocate
device memory (graph-capture regions, host callbacks, plugins whose host
framework owns all allocations).  It runs in a scratch area built into the
library with the same kernels in the same order as the workspace-based
nvfp4_linear_fwd, so Y must be bit-identical to that call's, call after call,
and the call must leave the device's free memory unchanged.

Named so that pytest collects it last; it must pass alone in a fresh process
and after the rest of the suite."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import _lib, api, synth
from tests._parity import sample_pairs

pytestmark = pytest.mark.gpu

SCRATCH = 16 << 20          # NVFP4_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_bit_microscaled_b200 import build
    build.build()
    return _lib.lib()


def _oracle_check(X, W, Y, pairs=None):
    """Y within the GEMM parity bound of the oracle's own quantization of X and
    W: |err| <= 1e-4 * sum_k |a_k b_k| + 2^-8 |D| (BF16 output)."""
    ax, aw = O.amax(X), O.amax(W)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), _ = O.expand_2d(cw, tw)
    D, absum = O.gemm(cx, sx, float(O.global_scales(ax)[1]), cwr, swr, float(O.global_scales(aw)[1]), pairs=pairs)
    got = Y.float().cpu().numpy().astype(np.float64)
    got = got if pairs is None else got[pairs[:, 0], pairs[:, 1]]
    bound = 1e-4 * absum + 2.0 ** -8 * np.abs(D) + 1e-30
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - D) <= bound), "outside the oracle bound"


@pytest.mark.parametrize("T,Cin,Cout,check_all", [(256, 512, 384, True), (16384, 512, 512, False)])
def test_noalloc_forward_equals_workspace_forward_two_calls_in_a_row(L, T, Cin, Cout, check_all):
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((301, 302)):          # two calls in a row, different inputs
        X = synth.activations(T, Cin, seed)
        W = synth.weights(Cout, Cin, seed)
        Xd, Wd = X.cuda(), W.cuda()
        ws = api.LinearWorkspace(T, Cin, Cout, "cuda")
        Y_ref = api.linear_fwd(Xd, Wd, ws)
        Y = torch.full((T, Cout), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st = L.nvfp4_linear_fwd_noalloc(Xd.data_ptr(), Wd.data_ptr(), T, Cin, Cout, Y.data_ptr(), stream)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        assert st == 0, f"call {call}: status {st}"
        assert free_after == free_before, f"call {call}: free device memory changed by {free_before - free_after} B"
        assert torch.equal(Y, Y_ref), f"call {call}: differs from nvfp4_linear_fwd"
        _oracle_check(X, W, Y, None if check_all else sample_pairs(T, Cout, 512, seed=call))


def test_noalloc_limit_counts_only_the_forward_operands(L):
    # the forward of this shape fits the scratch while the full forward+backward workspace does not
    T, Cin, Cout = 16384, 512, 512
    assert L.nvfp4_linear_workspace_bytes(T, Cin, Cout) > SCRATCH


def test_noalloc_rejects_sizes_beyond_its_scratch(L):
    T, Cin, Cout = 4096, 4096, 4096
    assert L.nvfp4_linear_workspace_bytes(T, Cin, Cout) > SCRATCH
    fake = 1 << 20                                     # never dereferenced: rejected first
    assert L.nvfp4_linear_fwd_noalloc(fake, fake, T, Cin, Cout, fake, None) == 7   # NVFP4_ERR_WORKSPACE
    assert L.nvfp4_linear_fwd_noalloc(fake, fake, 100, 64, 64, fake, None) == 2    # NVFP4_ERR_SHAPE
    assert L.nvfp4_linear_fwd_noalloc(fake, fake, 1 << 31, 64, 64, fake, None) == 2
