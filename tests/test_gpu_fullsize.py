"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (CTA-pair GEMM kernel, one-pass amax, the linear-layer C entry points,
and the data-parallel layer with its one-read ROWCOL quantizer and second
stream).

Every quantized operand is compared with the oracle byte for byte over the
whole tensor; GEMM outputs on 4096 seeded sampled entries (plus corners),
each within |err| <= 1e-4 * sum_k |a_k b_k| (+ 2^-8 |ref| for BF16 outputs)."""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_bit_microscaled_b200 import api, synth
from tests._parity import assert_gemm_close, assert_q_equal, sample_pairs

pytestmark = pytest.mark.gpu

NS = 4096


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


def _gs(a):
    return float(O.global_scales(a)[1])


def _check_sampled(D, ca, sa, ga, cb, sb, gb, bf16, what, seed):
    M, N = D.shape
    pairs = sample_pairs(M, N, NS, seed=seed)
    ref, absum = O.gemm(ca, sa, ga, cb, sb, gb, pairs=pairs)
    got = D[torch.from_numpy(pairs[:, 0]).cuda(), torch.from_numpy(pairs[:, 1]).cuda()].float().cpu().numpy()
    assert_gemm_close(got, ref, absum, bf16=bf16, what=what)


def test_fullsize_fprop_workload():
    # X 8192x5120 (0.1% outlier channels), W 20480x5120 ~N(0,0.02) 2D; Y = X W^T
    wl = synth.WORKLOADS["fprop"]
    T, Cin, Cout, seed = wl["T"], wl["Cin"], wl["Cout"], wl["seed"]
    Xd = synth.activations(T, Cin, seed, device="cuda")
    Wd = synth.weights(Cout, Cin, seed, device="cuda")
    X, W = Xd.cpu(), Wd.cpu()
    ax, aw = O.amax(X), O.amax(W)
    a_dev = api.amax(Xd)
    w_dev = api.amax(Wd)
    assert float(a_dev.cpu()[0]) == ax and float(w_dev.cpu()[0]) == aw
    xr, _ = api.quantize(Xd, api.ROW, a_dev)
    wr, wc = api.quantize(Wd, api.TWO_D, w_dev)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), (cwc, swc) = O.expand_2d(cw, tw)
    assert_q_equal(xr, cx, sx, ax, "X row")
    assert_q_equal(wr, cwr, swr, aw, "W 2D row")
    assert_q_equal(wc, cwc, swc, aw, "W 2D col")
    Y = api.gemm(xr, wr, api.OUT_BF16)
    _check_sampled(Y, cx, sx, _gs(ax), cwr, swr, _gs(aw), True, "fprop Y", 11)
    # the same GEMM with the amax of Y reduced in its epilogue
    Y2, amax_y = api.gemm_amax(xr, wr, api.OUT_BF16)
    assert torch.equal(Y2, Y)
    assert float(amax_y.cpu()[0]) == float(Y.float().abs().max().cpu()) == float(api.amax(Y).cpu()[0])


def test_fullsize_wgrad_workload():
    # dY 8192x20480 ~N(0,1e-3) x row lognormal; RHT + SR (seed 1) on dY, RHT on X; dW = dY^T X
    wl = synth.WORKLOADS["wgrad"]
    T, Cin, Cout, seed = wl["T"], wl["Cin"], wl["Cout"], wl["seed"]
    Xd = synth.activations(T, Cin, seed, device="cuda")
    Gd = synth.gradients(T, Cout, seed, device="cuda")
    X, G = Xd.cpu(), Gd.cpu()
    xb = api.amax(Xd, rht=2).cpu().numpy()
    gb = api.amax(Gd, rht=2).cpu().numpy()
    axr, agr = O.amax_rht(X), O.amax_rht(G)
    assert xb[0] == O.amax(X) and xb[1] == axr and gb[0] == O.amax(G) and gb[1] == agr
    _, xc = api.quantize(Xd, api.COL, api.amax(Xd, rht=True), rht=True)
    _, gc = api.quantize(Gd, api.COL, api.amax(Gd, rht=True), rht=True, sr=True, seed=1)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    cgc, sgc = O.quantize_col(G, agr, rht=True, sr=True, seed=1)
    assert_q_equal(xc, cxc, sxc, axr, "X col RHT")
    assert_q_equal(gc, cgc, sgc, agr, "dY col RHT SR")
    dW = api.gemm(gc, xc, api.OUT_F32)
    _check_sampled(dW, cgc, sgc, _gs(agr), cxc, sxc, _gs(axr), False, "wgrad dW", 12)


def test_fullsize_linear_layer():
    # T = 16384, 5120 -> 20480, fwd + bwd through nvfp4_linear_fwd / nvfp4_linear_bwd (seed 2)
    wl = synth.WORKLOADS["full"]
    T, Cin, Cout, seed = wl["T"], wl["Cin"], wl["Cout"], wl["seed"]
    Xd, Wd, Gd = synth.workload_inputs("full", device="cuda")
    ws = api.LinearWorkspace(T, Cin, Cout, "cuda")
    Y = api.linear_fwd(Xd, Wd, ws)
    dX, dW = api.linear_bwd(Gd, ws, seed)
    torch.cuda.synchronize()
    X, W, G = Xd.cpu(), Wd.cpu(), Gd.cpu()
    ax, axr, aw, ag, agr = O.amax(X), O.amax_rht(X), O.amax(W), O.amax(G), O.amax_rht(G)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), (cwc, swc) = O.expand_2d(cw, tw)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    cg, sg = O.quantize_row(G, ag, sr=True, seed=seed)
    cgc, sgc = O.quantize_col(G, agr, rht=True, sr=True, seed=seed)
    for name, codes, sf, a in (("x_row", cx, sx, ax), ("w_row", cwr, swr, aw), ("w_col", cwc, swc, aw),
                               ("x_col", cxc, sxc, axr), ("dy_row", cg, sg, ag), ("dy_col", cgc, sgc, agr)):
        assert_q_equal(ws.tensor(name), codes, sf, a, name)
    _check_sampled(Y, cx, sx, _gs(ax), cwr, swr, _gs(aw), True, "Y", 21)
    _check_sampled(dX, cg, sg, _gs(ag), cwc, swc, _gs(aw), True, "dX", 22)
    _check_sampled(dW, cgc, sgc, _gs(agr), cxc, sxc, _gs(axr), False, "dW", 23)


def test_fullsize_large_outlier_workload():
    # X 32768x8192 Student-t(3), W 8192^2 with 0.01% entries x50, dY 32768x8192 ~N(0,1e-3)
    wl = synth.WORKLOADS["large"]
    T, Cin, Cout, seed = wl["T"], wl["Cin"], wl["Cout"], wl["seed"]
    Xd, Wd, Gd = synth.workload_inputs("large", device="cuda")
    X, W, G = Xd.cpu(), Wd.cpu(), Gd.cpu()
    ax, aw, ag = O.amax(X), O.amax(W), O.amax(G)
    axr, agr = O.amax_rht(X), O.amax_rht(G)
    xa, wa, ga = api.amax(Xd, rht=2), api.amax(Wd), api.amax(Gd, rht=2)
    assert list(xa.cpu().numpy()) == [ax, axr] and float(wa.cpu()[0]) == aw
    assert list(ga.cpu().numpy()) == [ag, agr]
    xr, _ = api.quantize(Xd, api.ROW, xa[0:1])
    wr, wc = api.quantize(Wd, api.TWO_D, wa)
    gr, _ = api.quantize(Gd, api.ROW, ga[0:1], sr=True, seed=seed)
    _, gc = api.quantize(Gd, api.COL, ga[1:2], rht=True, sr=True, seed=seed)
    _, xc = api.quantize(Xd, api.COL, xa[1:2], rht=True)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), (cwc, swc) = O.expand_2d(cw, tw)
    cg, sg = O.quantize_row(G, ag, sr=True, seed=seed)
    cgc, sgc = O.quantize_col(G, agr, rht=True, sr=True, seed=seed)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    assert_q_equal(xr, cx, sx, ax, "X row")
    assert_q_equal(wr, cwr, swr, aw, "W row")
    assert_q_equal(wc, cwc, swc, aw, "W col")
    assert_q_equal(gr, cg, sg, ag, "dY row SR")
    assert_q_equal(gc, cgc, sgc, agr, "dY col RHT SR")
    assert_q_equal(xc, cxc, sxc, axr, "X col RHT")
    _check_sampled(api.gemm(xr, wr, api.OUT_BF16), cx, sx, _gs(ax), cwr, swr, _gs(aw), True, "fprop", 31)
    _check_sampled(api.gemm(gr, wc, api.OUT_BF16), cg, sg, _gs(ag), cwc, swc, _gs(aw), True, "dgrad", 32)
    _check_sampled(api.gemm(gc, xc, api.OUT_F32), cgc, sgc, _gs(agr), cxc, sxc, _gs(axr), False, "wgrad", 33)
    # the launch configuration bench.py times: the data-parallel layer on one rank, with X's
    # one-read ROWCOL quantizer and the second stream (W's branch, the dY row copy beside wgrad)
    from nvfp4_bit_microscaled_b200.dp import DataParallelLinear
    layer = DataParallelLinear(T, Cin, Cout, "cuda")
    Y = layer.forward(Xd, Wd)
    dX, dW = layer.backward(Gd, seed)
    torch.cuda.synchronize()
    assert list(layer.amax_x.cpu().numpy()) == [ax, axr] and list(layer.amax_dy.cpu().numpy()) == [ag, agr]
    for q, codes, sf, a, name in ((layer.x_row, cx, sx, ax, "layer X row"), (layer.x_col, cxc, sxc, axr, "layer X col"),
                                  (layer.w_row, cwr, swr, aw, "layer W row"), (layer.w_col, cwc, swc, aw, "layer W col"),
                                  (layer.dy_row, cg, sg, ag, "layer dY row"), (layer.dy_col, cgc, sgc, agr, "layer dY col")):
        assert_q_equal(q, codes, sf, a, name)
    _check_sampled(Y, cx, sx, _gs(ax), cwr, swr, _gs(aw), True, "layer Y", 34)
    _check_sampled(dX, cg, sg, _gs(ag), cwc, swc, _gs(aw), True, "layer dX", 35)
    _check_sampled(dW, cgc, sgc, _gs(agr), cxc, sxc, _gs(axr), False, "layer dW", 36)
