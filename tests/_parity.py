"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the CPU oracle on the same BF16 bytes, compare."""
import numpy as np
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import api

GEMM_REL = 1e-4          # |err| <= 1e-4 * sum_k |a_k b_k|
BF16_REL = 2.0 ** -8     # extra relative slack when the output is BF16


def q_numpy(q):
    """GPU QTensor -> (packed data [rows, cols/2], swizzled scales, s_g)."""
    return (q.data.cpu().numpy(), q.scales.cpu().numpy(), float(q.global_scale.cpu()[0]))


def assert_q_equal(q, codes, sf, amax, what=""):
    """Bit-exact: packed codes, swizzled scales (padding included) and s_g."""
    data, scales, sg = q_numpy(q)
    want_data = O.pack_nibbles(codes)
    want_sf = O.swizzle_scales(sf)
    if not np.array_equal(data, want_data):
        bad = np.argwhere(data != want_data)
        r, c = bad[0]
        raise AssertionError(f"{what}: {len(bad)} code bytes differ; first at row {r} byte {c}: "
                             f"gpu {data[r, c]:#04x} oracle {want_data[r, c]:#04x}")
    if not np.array_equal(scales, want_sf):
        bad = np.flatnonzero(scales != want_sf)
        raise AssertionError(f"{what}: {len(bad)} scale bytes differ; first at offset {bad[0]}: "
                             f"gpu {scales[bad[0]]:#04x} oracle {want_sf[bad[0]]:#04x}")
    want_sg = float(O.global_scales(amax)[1])
    assert sg == want_sg or (np.isnan(sg) and np.isnan(want_sg)), what


def assert_gemm_close(D_gpu, D_ref, absum, bf16=False, what=""):
    D_gpu = np.asarray(D_gpu, dtype=np.float64)
    tol = GEMM_REL * absum + (BF16_REL * np.abs(D_ref) if bf16 else 0.0) + 1e-30
    err = np.abs(D_gpu - D_ref)
    bad = err > tol
    if bad.any():
        i = np.flatnonzero(bad.ravel())[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} entries outside the bound; first flat index {i}: "
                             f"gpu {D_gpu.ravel()[i]!r} ref {D_ref.ravel()[i]!r} bound {tol.ravel()[i]!r}")
    assert np.all(np.isfinite(D_gpu)), what


def sample_pairs(M, N, n, seed=0):
    rng = np.random.default_rng(seed)
    pairs = np.stack([rng.integers(0, M, n), rng.integers(0, N, n)], axis=1)
    # always include the corners and the last row/column (ragged tails)
    extra = np.array([[0, 0], [M - 1, N - 1], [0, N - 1], [M - 1, 0]])
    return np.concatenate([extra, pairs]).astype(np.int64)


def dev(x):
    return x.to("cuda").contiguous()


def gpu_amax(x, rht=False):
    return float(api.amax(dev(x), rht=rht).cpu()[0])


def cpu(x):
    return x.detach().to("cpu")


__all__ = ["q_numpy", "assert_q_equal", "assert_gemm_close", "sample_pairs", "dev", "gpu_amax",
           "cpu", "torch"]
