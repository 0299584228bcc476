"""Row blocks of a tensor (nvfp4_quantize_rows) and the data-parallel linear
layer (nvfp4_bit_microscaled_b200.dp) on the GPU.

- A row block quantized with its global row offset equals the matching slice
  of the oracle's quantization of the whole tensor, bit for bit, with SR on
  and off, for the row copy and the RHT column copy.
- Two ranks on one GPU (gloo, whose collectives run on the host; no kernel
  of one rank waits on the other) run the DP layer on their halves of a
  batch.  Y, dX and every quantized copy equal the one-process
  nvfp4_linear_fwd/bwd results on the whole batch; dW lies within the GEMM
  bound of the oracle's whole-batch wgrad."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

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


@pytest.mark.parametrize("row0,rows", [(0, 96), (96, 128), (160, 96), (48, 208)])
@pytest.mark.parametrize("sr", [False, True])
def test_row_block_equals_slice_of_whole(row0, rows, sr):
    R, C, seed = 256, 320, 21
    x = synth.gradients(R, C, 31)
    a, ar = O.amax(x), O.amax_rht(x)
    blk = dev(x)[row0:row0 + rows]
    a_dev = torch.tensor([a], dtype=torch.float32, device="cuda")
    ar_dev = torch.tensor([ar], dtype=torch.float32, device="cuda")
    qr, _ = api.quantize(blk, api.ROW, a_dev, sr=sr, seed=seed, row0=row0)
    _, qc = api.quantize(blk, api.COL, ar_dev, rht=True, sr=sr, seed=seed, row0=row0)
    codes, sf = O.quantize_row(x, a, sr=sr, seed=seed)
    assert_q_equal(qr, codes[row0:row0 + rows], sf[row0:row0 + rows], a, f"rows {row0}+{rows}")
    ccodes, csf = O.quantize_col(x, ar, rht=True, sr=sr, seed=seed)
    assert_q_equal(qc, ccodes[:, row0:row0 + rows], csf[:, row0 // 16:(row0 + rows) // 16], ar,
                   f"cols {row0}+{rows}")


WORLD = 2
T, CIN, COUT, SEED = 512, 256, 384, 13


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch():
    return synth.activations(T, CIN, 41), synth.weights(COUT, CIN, 42, std=0.02), synth.gradients(T, COUT, 43)


def _rank(rank, port, out_dir):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from nvfp4_bit_microscaled_b200 import dp

    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    X, W, dY = _batch()
    tl = T // WORLD
    rows = slice(rank * tl, (rank + 1) * tl)
    layer = dp.DataParallelLinear(tl, CIN, COUT, "cuda")
    Y = layer.forward(X[rows].contiguous().cuda(), W.cuda())
    dX, dW = layer.backward(dY[rows].contiguous().cuda(), SEED)
    torch.cuda.synchronize()
    out = {"Y": Y.cpu(), "dX": dX.cpu(), "dW": dW.cpu()}
    for name in ("x_row", "x_col", "dy_row", "dy_col"):
        q = getattr(layer, name)
        out[name] = (q.data.cpu(), q.scales.cpu())
    torch.save(out, os.path.join(out_dir, f"rank{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


def _unswizzle(scales, rows, S):
    """[rows, S] scale matrix out of the 128x4-tile byte layout."""
    Sp = (S + 3) // 4 * 4
    r = np.arange(rows)[:, None]
    c = np.arange(S)[None, :]
    off = ((r // 128) * (Sp // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return scales.numpy()[off]


def test_data_parallel_linear_two_ranks_equal_one_process(tmp_path):
    mp.spawn(_rank, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    X, W, dY = _batch()
    ws = api.LinearWorkspace(T, CIN, COUT, "cuda")
    Y = api.linear_fwd(X.cuda(), W.cuda(), ws)
    dX, dW = api.linear_bwd(dY.cuda(), ws, SEED)
    torch.cuda.synchronize()
    tl = T // WORLD
    whole = {name: ws.tensor(name) for name in ("x_row", "x_col", "dy_row", "dy_col")}
    for rank in range(WORLD):
        got = torch.load(tmp_path / f"rank{rank}.pt")
        rows = slice(rank * tl, (rank + 1) * tl)
        assert torch.equal(got["Y"], Y[rows].cpu()), rank
        assert torch.equal(got["dX"], dX[rows].cpu()), rank
        for name in ("x_row", "dy_row"):       # [tokens, C]: rows of the whole copy
            data, sc = got[name]
            q = whole[name]
            assert torch.equal(data, q.data[rows].cpu()), name
            S = q.cols // 16
            assert np.array_equal(_unswizzle(sc, tl, S), _unswizzle(q.scales.cpu(), T, S)[rows]), name
        for name in ("x_col", "dy_col"):       # [C, tokens]: token columns of the whole copy
            data, sc = got[name]
            q = whole[name]
            assert torch.equal(data, q.data[:, rank * tl // 2:(rank + 1) * tl // 2].cpu()), name
            blocks = slice(rank * tl // 16, (rank + 1) * tl // 16)
            assert np.array_equal(_unswizzle(sc, q.rows, tl // 16),
                                  _unswizzle(q.scales.cpu(), q.rows, T // 16)[:, blocks]), name
    # dW: the two partial wgrads summed, within the GEMM bound of the whole-batch oracle
    agr, axr = O.amax_rht(dY), O.amax_rht(X)
    gs = lambda a: float(O.global_scales(a)[1])
    cgc, sgc = O.quantize_col(dY, agr, rht=True, sr=True, seed=SEED)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    ref, absum = O.gemm(cgc, sgc, gs(agr), cxc, sxc, gs(axr))
    # each partial is within 1e-4 of its own sum of |a b|, so their sum is within 1e-4 * absum; the
    # final FP32 addition of the two partials adds one rounding (2^-24 relative, taken as 2^-22)
    tol = 1e-4 * absum + 2.0 ** -22 * np.abs(ref) + 1e-30
    for rank in range(WORLD):
        got = torch.load(tmp_path / f"rank{rank}.pt")["dW"].numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= tol), f"dW rank {rank}: {np.sum(np.abs(got - ref) > tol)} outside"


@pytest.mark.parametrize("row0", [(1 << 36) // 320 - 16, (1 << 36) // 320 + 16, 1 << 32])
def test_row_block_past_index_2_36(row0):
    # the block counters (element index / 16) of these rows pass 2^32 (the
    # first row block straddles it), so the launchers pick the general SR
    # kernels, whose Philox counter keeps a high word; codes and scales must
    # equal the oracle's for the same offset
    row0 -= row0 % 16
    x = synth.gradients(64, 320, 43)
    a, ar = O.amax(x), O.amax_rht(x)
    xd = dev(x)
    a_dev, ar_dev = api.amax(xd), api.amax(xd, rht=True)
    assert row0 * 320 + 64 * 320 >= 1 << 36
    qr, _ = api.quantize(xd, api.ROW, a_dev, sr=True, seed=11, row0=row0)
    assert_q_equal(qr, *O.quantize_row(x, a, sr=True, seed=11, row0=row0), a, f"row sr row0={row0}")
    _, qc = api.quantize(xd, api.COL, a_dev, sr=True, seed=11, row0=row0)
    assert_q_equal(qc, *O.quantize_col(x, a, sr=True, seed=11, row0=row0), a, f"col sr row0={row0}")
    _, qcr = api.quantize(xd, api.COL, ar_dev, rht=True, sr=True, seed=11, row0=row0)
    assert_q_equal(qcr, *O.quantize_col(x, ar, rht=True, sr=True, seed=11, row0=row0), ar,
                   f"col rht sr row0={row0}")
