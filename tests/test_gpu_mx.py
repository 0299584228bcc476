"""MXFP4 comparison format on the GPU vs the oracle (readings R21-R24):
row-wise 1x32 quantization bit for bit (codes, UE8M0 scales, padding) and the
block-32 CTA-pair GEMM within |err| <= 1e-4 * sum_k |a_k b_k| (+ 2^-8 |ref| for
BF16 output), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import api, synth
from tests._parity import assert_gemm_close, dev, sample_pairs

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


def _assert_mx_equal(q, codes, sf, what):
    got_data = q.data.cpu().numpy()
    want_data = O.pack_nibbles(codes)
    bad = np.argwhere(got_data != want_data)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ, first {bad[:3].tolist()}"
    got_sf = q.scales.cpu().numpy()
    want_sf = O.swizzle_scales(sf)
    assert got_sf.shape == want_sf.shape, what
    bad = np.flatnonzero(got_sf != want_sf)
    assert bad.size == 0, f"{what}: {bad.size} scale bytes differ, first {bad[:3].tolist()}"
    assert float(q.global_scale.cpu()[0]) == 1.0


def _extremes():
    # zero blocks, BF16 subnormals (scale clamps at 2^-127), huge values, exact
    # midpoints and values that saturate to 6 * 2^s
    x = np.zeros((4, 128), dtype=np.float32)
    x[1, :32] = np.float32(2.0 ** -133) * np.arange(1, 33)
    x[2, 32:64] = 2.0 ** 120 * np.linspace(-7.5, 7.5, 32)
    x[3, 64:96] = [7.0, 3.5, 2.5, 0.75, 0.25, -5.0, -0.25, 1.25] * 4
    x[3, 96:] = np.linspace(-1e-3, 1e-3, 32)
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("name,x", [
    ("tiny_x", synth.workload_inputs("tiny")[0]),
    ("act_outliers", synth.activations(256, 640, 21)),
    ("grad_lognormal", synth.gradients(272, 320, 22)),
    ("heavy_t3", synth.heavy_activations(144, 192, 23)),
    ("weights_partial_word", synth.weights(208, 96, 24, std=0.02)),    # 3 blocks: partial scale word
    ("extremes", _extremes()),
])
def test_mx_quantize_row_bit_exact(name, x):
    q = api.mx_quantize(dev(x))
    codes, sf = O.mx_quantize_row(x)
    _assert_mx_equal(q, codes, sf, name)


def test_mx_quantize_strided_rows():
    big = synth.activations(64, 320, 25)
    view = dev(big)[:, 32:288]
    q = api.mx_quantize(view)
    codes, sf = O.mx_quantize_row(big[:, 32:288].contiguous())
    _assert_mx_equal(q, codes, sf, "strided")


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (512, 768, 1280), (256, 512, 64), (768, 256, 320),
                                   (2304, 1536, 512), (256, 256, 96), (512, 256, 160),
                                   (200, 272, 320), (96, 48, 128), (1000, 528, 256)])   # M, N tails
@pytest.mark.parametrize("bf16", [False, True])
def test_mx_gemm_vs_oracle(M, N, K, bf16):
    xa = synth.activations(M, K, 71)
    xb = synth.weights(N, K, 72, std=0.02)
    qa, qb = api.mx_quantize(dev(xa)), api.mx_quantize(dev(xb))
    ca, sa = O.mx_quantize_row(xa)
    cb, sb = O.mx_quantize_row(xb)
    _assert_mx_equal(qa, ca, sa, "A")
    _assert_mx_equal(qb, cb, sb, "B")
    D = api.mx_gemm(qa, qb, api.OUT_BF16 if bf16 else api.OUT_F32).float().cpu().numpy()
    if M * N <= 1 << 20:
        ref, absum = O.mx_gemm(ca, sa, cb, sb)
        assert_gemm_close(D, ref, absum, bf16=bf16, what=f"mx {M}x{N}x{K}")
    else:
        pairs = sample_pairs(M, N, 8192, seed=6)
        ref, absum = O.mx_gemm(ca, sa, cb, sb, pairs=pairs)
        assert_gemm_close(D[pairs[:, 0], pairs[:, 1]], ref, absum, bf16=bf16, what=f"mx {M}x{N}x{K}")


def test_mx_gemm_one_block_per_row_pins_scale_byte_pairs():
    # A row m is zero except K-block j(m) = m % (K/32), whose 32 codes are 1.0
    # with scale 2^(m % 5); B is 1.0 everywhere with block scale 2^(block % 7).
    # D[m, n] = 32 * 2^(m % 5) * 2^(j(m) % 7) exposes any mix-up of the byte
    # pair a K=64 step reads from its scale cell.
    M, N, K = 256, 256, 512
    S = K // 32
    ca = np.zeros((M, K), np.uint8)
    sa = np.full((M, S), 127, np.uint8)
    for m in range(M):
        j = m % S
        ca[m, 32 * j:32 * j + 32] = 2                        # code 2 = 1.0
        sa[m, j] = 127 + m % 5
    cb = np.full((N, K), 2, np.uint8)
    sb = np.tile((127 + np.arange(S) % 7).astype(np.uint8), (N, 1))

    def qt(codes, sf):
        rows = codes.shape[0]
        return api.QTensor(torch.from_numpy(O.pack_nibbles(codes)).cuda(),
                           torch.from_numpy(O.swizzle_scales(sf)).cuda(),
                           torch.ones(1, device="cuda"), rows, K)

    D = api.mx_gemm(qt(ca, sa), qt(cb, sb)).cpu().numpy()
    want = np.array([[32.0 * 2.0 ** (m % 5) * 2.0 ** ((m % S) % 7)] * N for m in range(M)])
    assert np.array_equal(D, want)
    ref, _ = O.mx_gemm(ca, sa, cb, sb)
    assert np.array_equal(ref, want)
