"""nvfp4_linear_fwd_noalloc: the linear forward for callers that cannot allocate
device memory (graph-capture regions, host callbacks, plugins whose host
framework owns all allocations).  It runs in a scratch area built into the
library, so its output must equal the workspace-based nvfp4_linear_fwd's on
the same inputs, call after call.

Named so that pytest collects it last; it must pass alone in a fresh process
and after the rest of the suite."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_bit_microscaled_b200 import build
    build.build()
    return _lib.lib()


def _gemm_bound(X, W):
    """Per-entry bound used by the GEMM parity tests, from the oracle's own
    quantization of X and W: 1e-4 * sum_k |a_k b_k| + 2^-8 |D| for BF16 output."""
    ax, aw = O.amax(X), O.amax(W)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), _ = O.expand_2d(cw, tw)
    D, absum = O.gemm(cx, sx, float(O.global_scales(ax)[1]), cwr, swr, float(O.global_scales(aw)[1]))
    return D, 1e-4 * absum + 2.0 ** -8 * np.abs(D) + 1e-30


def test_noalloc_forward_matches_workspace_forward_two_calls_in_a_row(L):
    T, Cin, Cout = 256, 512, 384
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((301, 302)):          # two calls, different inputs
        X = synth.activations(T, Cin, seed)
        W = synth.weights(Cout, Cin, seed)
        Xd, Wd = X.cuda(), W.cuda()
        ws = api.LinearWorkspace(T, Cin, Cout, "cuda")
        Y_ref = api.linear_fwd(Xd, Wd, ws)
        Y = torch.full((T, Cout), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = L.nvfp4_linear_fwd_noalloc(Xd.data_ptr(), Wd.data_ptr(), T, Cin, Cout, Y.data_ptr(), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        D, bound = _gemm_bound(X, W)
        got = Y.float().cpu().numpy().astype(np.float64)
        ref = Y_ref.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {call}"
        assert np.all(np.abs(got - ref) <= bound), f"call {call}: differs from nvfp4_linear_fwd"
        assert np.all(np.abs(got - D) <= bound), f"call {call}: outside the oracle bound"


def test_noalloc_rejects_sizes_beyond_its_scratch(L):
    limit = 16 << 20
    T, Cin, Cout = 4096, 4096, 4096
    assert L.nvfp4_linear_workspace_bytes(T, Cin, Cout) > limit
    fake = 1 << 20                                     # never dereferenced: rejected first
    assert L.nvfp4_linear_fwd_noalloc(fake, fake, T, Cin, Cout, fake, None) == 7   # NVFP4_ERR_WORKSPACE
    assert L.nvfp4_linear_fwd_noalloc(fake, fake, 100, 64, 64, fake, None) == 2    # NVFP4_ERR_SHAPE
