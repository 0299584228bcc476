"""The data-parallel linear layer (nvfp4_bit_microscaled_b200.dp) on
world-size-2 gloo ranks, CPU only.

The module's calls into the library are replaced by the CPU oracle
(``_OracleApi``), so this checks the module's own logic: which amax feeds
which copy, the MAX all-reduce of the amaxes, the global row offset of the
SR draws, and the SUM all-reduce of dW.  A row block is quantized by the
oracle as the bottom rows of a tensor whose first row0 rows are zero: the
blocks never straddle row0 (row0 % 16 == 0), and the SR draws are then keyed
by the whole-tensor index, which is what nvfp4_quantize_rows promises.

Expected values come from the oracle on the whole batch: each rank's
quantized copies must be slices of it, Y and dX its rows, and dW its FP64
result up to the order of the two-rank sum."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2
T, CIN, COUT, SEED = 64, 48, 80, 11


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    from nvfp4_bit_microscaled_b200 import synth
    return synth.activations(T, CIN, 4), synth.weights(COUT, CIN, 5, std=0.02), synth.gradients(T, COUT, 6)


class _Q:
    def __init__(self, rows, cols):
        self.rows, self.cols = rows, cols
        self.codes = self.sf = None
        self.gs = None


class _OracleApi:
    """The subset of nvfp4_bit_microscaled_b200.api that dp.py calls, on the oracle."""
    ROW, COL, ROWCOL, TWO_D = 1, 2, 3, 4
    OUT_F32, OUT_BF16 = 0, 1

    def __init__(self, O):
        self.O = O

    def empty_qtensor(self, rows, cols, device):
        return _Q(rows, cols)

    def amax(self, x, rht=False, out=None):
        vals = {0: [self.O.amax(x)], 1: [self.O.amax_rht(x)], 2: [self.O.amax(x), self.O.amax_rht(x)]}[int(rht)]
        out.copy_(torch.tensor(vals, dtype=torch.float32))
        return out

    def _padded(self, x, row0):
        return torch.cat([torch.zeros(row0, x.shape[1], dtype=x.dtype), x]) if row0 else x

    def quantize(self, x, mode, amax_dev, rht=False, sr=False, seed=0, row_out=None, col_out=None, row0=0):
        O, a = self.O, float(amax_dev[0])
        R = x.shape[0]
        gs = float(O.global_scales(a)[1])
        if mode == self.TWO_D:
            cw, tw = O.quantize_2d(x, a)
            (row_out.codes, row_out.sf), (col_out.codes, col_out.sf) = O.expand_2d(cw, tw)
            row_out.gs = col_out.gs = gs
            return row_out, col_out
        xp = self._padded(x, row0)
        if mode in (self.ROW, self.ROWCOL):
            c, s = O.quantize_row(xp, a, sr=sr, seed=seed)
            row_out.codes, row_out.sf, row_out.gs = c[row0:], s[row0:], gs
            assert row_out.codes.shape[0] == R
        if mode in (self.COL, self.ROWCOL):
            # ROWCOL with RHT: the column copy is scaled by the second amax (the RHT one)
            ac = float(amax_dev[1]) if (mode == self.ROWCOL and rht) else a
            c, s = O.quantize_col(xp, ac, rht=rht, sr=sr, seed=seed)
            col_out.codes, col_out.sf, col_out.gs = c[:, row0:], s[:, row0 // 16:], float(O.global_scales(ac)[1])
            assert col_out.codes.shape[1] == R
        return row_out, col_out

    def gemm(self, A, B, out_dtype=0, out=None):
        D, _ = self.O.gemm(A.codes, A.sf, A.gs, B.codes, B.sf, B.gs)
        return torch.from_numpy(D)


def _worker(rank, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    from nvfp4_bit_microscaled_b200 import dp

    if port is not None:                 # mp.spawn; under torchrun the launcher set MASTER_*
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    dp.api = _OracleApi(O)
    X, W, dY = _inputs()
    tl = T // WORLD
    rows = slice(rank * tl, (rank + 1) * tl)
    layer = dp.DataParallelLinear(tl, CIN, COUT, "cpu")
    Y = layer.forward(X[rows].contiguous(), W)
    dX, dW = layer.backward(dY[rows].contiguous(), SEED)
    save = dict(Y=Y.numpy(), dX=dX.numpy(), dW=dW.numpy(), amax_x=layer.amax_x.numpy(),
                amax_dy=layer.amax_dy.numpy())
    for name in ("x_row", "x_col", "dy_row", "dy_col"):
        q = getattr(layer, name)
        save[name + "_codes"], save[name + "_sf"] = q.codes, q.sf
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **save)
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_linear_equals_whole_batch(tmp_path):
    mp.spawn(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    _check(tmp_path)


def test_data_parallel_linear_under_torchrun(tmp_path):
    # the launch the multi-GPU bench uses: torchrun, one process per rank, env:// rendezvous
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", str(WORLD),
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.abspath(__file__),
           str(tmp_path)]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    _check(tmp_path)


def _check(tmp_path):
    import oracle as O
    X, W, dY = _inputs()
    ax, axr, ag, agr = O.amax(X), O.amax_rht(X), O.amax(dY), O.amax_rht(dY)
    gs = lambda a: float(O.global_scales(a)[1])
    cx, sx = O.quantize_row(X, ax)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    cg, sg = O.quantize_row(dY, ag, sr=True, seed=SEED)
    cgc, sgc = O.quantize_col(dY, agr, rht=True, sr=True, seed=SEED)
    cw, tw = O.quantize_2d(W, O.amax(W))
    (cwr, swr), (cwc, swc) = O.expand_2d(cw, tw)
    Y, _ = O.gemm(cx, sx, gs(ax), cwr, swr, gs(O.amax(W)))
    dX, _ = O.gemm(cg, sg, gs(ag), cwc, swc, gs(O.amax(W)))
    dW, absum = O.gemm(cgc, sgc, gs(agr), cxc, sxc, gs(axr))
    tl = T // WORLD
    for rank in range(WORLD):
        r = np.load(tmp_path / f"rank{rank}.npz")
        rows, blocks = slice(rank * tl, (rank + 1) * tl), slice(rank * tl // 16, (rank + 1) * tl // 16)
        assert np.array_equal(r["amax_x"], np.array([ax, axr], np.float32))      # MAX over the ranks
        assert np.array_equal(r["amax_dy"], np.array([ag, agr], np.float32))
        assert np.array_equal(r["x_row_codes"], cx[rows]) and np.array_equal(r["x_row_sf"], sx[rows])
        assert np.array_equal(r["x_col_codes"], cxc[:, rows]) and np.array_equal(r["x_col_sf"], sxc[:, blocks])
        assert np.array_equal(r["dy_row_codes"], cg[rows]) and np.array_equal(r["dy_row_sf"], sg[rows])
        assert np.array_equal(r["dy_col_codes"], cgc[:, rows]) and np.array_equal(r["dy_col_sf"], sgc[:, blocks])
        assert np.array_equal(r["Y"], Y[rows]) and np.array_equal(r["dX"], dX[rows])
        assert np.all(np.abs(r["dW"] - dW) <= 1e-12 * absum + 1e-300)           # sum of two partial FP64 GEMMs


if __name__ == "__main__":        # one rank under torchrun (test_data_parallel_linear_under_torchrun)
    import sys
    _worker(int(os.environ["RANK"]), None, sys.argv[1])
