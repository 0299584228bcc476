"""Non-finite inputs (reading R25) on the CUDA path against the oracle: the amax
of a tensor holding a NaN is NaN and of one holding an infinity +inf; the RHT
amax of either is NaN; a quantizer handed a non-finite amax flags the copy
(every block scale 0x7F, every code 0, a non-finite decode scale), and a GEMM
that reads a flagged copy returns NaN.  The host sees the flag through
api.copy_is_flagged."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import api, synth
from tests._parity import assert_q_equal, dev

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


def _same(a, b):
    return (math.isnan(a) and math.isnan(b)) or a == b


def _planted(kind, R=96, C=160, seed=41):
    x = synth.activations(R, C, seed)
    x[37, 21] = {"inf": float("inf"), "-inf": float("-inf"), "nan": float("nan")}[kind]
    return x


@pytest.mark.parametrize("kind", ["inf", "-inf", "nan"])
def test_amax_of_nonfinite_tensor(kind):
    x = _planted(kind)
    a = api.amax(dev(x)).cpu().numpy()
    ar = api.amax(dev(x), rht=True).cpu().numpy()
    both = api.amax(dev(x), rht=2).cpu().numpy()
    assert _same(float(a[0]), O.amax(x)) and _same(float(both[0]), O.amax(x))
    assert math.isnan(float(ar[0])) and math.isnan(float(both[1])) and math.isnan(O.amax_rht(x))
    assert not math.isfinite(float(a[0]))


@pytest.mark.parametrize("kind", ["inf", "nan"])
def test_quantizers_flag_copies_of_nonfinite_tensor(kind):
    x = _planted(kind)
    xd = dev(x)
    a, ar = O.amax(x), O.amax_rht(x)
    a_dev, ar_dev = api.amax(xd), api.amax(xd, rht=True)
    row, _ = api.quantize(xd, api.ROW, a_dev)
    assert_q_equal(row, *O.quantize_row(x, a), a, "row")
    row_sr, _ = api.quantize(xd, api.ROW, a_dev, sr=True, seed=9)
    assert_q_equal(row_sr, *O.quantize_row(x, a, sr=True, seed=9), a, "row sr")
    _, col = api.quantize(xd, api.COL, ar_dev, rht=True, sr=True, seed=9)
    assert_q_equal(col, *O.quantize_col(x, ar, rht=True, sr=True, seed=9), ar, "col rht sr")
    rr, rc = api.quantize(xd, api.ROWCOL, api.amax(xd, rht=2), rht=True)
    assert_q_equal(rr, *O.quantize_row(x, a), a, "rowcol row")
    assert_q_equal(rc, *O.quantize_col(x, ar, rht=True), ar, "rowcol col")
    r2, c2 = api.quantize(xd, api.TWO_D, a_dev)
    (cr, sr_), (cc, sc) = O.expand_2d(*O.quantize_2d(x, a))
    assert_q_equal(r2, cr, sr_, a, "2d row")
    assert_q_equal(c2, cc, sc, a, "2d col")
    for q in (row, row_sr, col, rr, rc, r2, c2):
        assert api.copy_is_flagged(q)
        assert int((q.scales == 0x7F).sum()) == q.rows * (q.cols // 16)   # padding stays 0


def test_gemm_of_flagged_copy_is_nan_and_finite_copies_are_not_flagged():
    x = _planted("inf", R=128, C=256)
    w = synth.weights(128, 256, 42)
    qx, _ = api.quantize(dev(x), api.ROW, api.amax(dev(x)))
    qw, _ = api.quantize(dev(w), api.ROW, api.amax(dev(w)))
    assert api.copy_is_flagged(qx) and not api.copy_is_flagged(qw)
    D = api.gemm(qx, qw, api.OUT_F32)
    assert torch.isnan(D).all()
