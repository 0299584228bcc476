"""Data-parallel logic of the linear layer on world-size-2 gloo ranks (CPU).

Tokens shard across ranks.  With the activation amax all-reduced (MAX) before
quantization, each rank's round-to-nearest copies equal the matching slice of
a single-process quantization bit for bit, and the all-reduced partial wgrad
equals the full-batch wgrad.  Every rank computes with the CPU oracle; no GPU
is involved.  Also checks bench.py's max-over-ranks timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2
T, CIN, COUT = 128, 64, 96


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    from nvfp4_bit_microscaled_b200 import synth
    return synth.activations(T, CIN, 3), synth.gradients(T, COUT, 3)


def _worker(rank, port, out_dir):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    X, dY = _inputs()
    rows = slice(rank * T // WORLD, (rank + 1) * T // WORLD)
    Xs, dYs = X[rows].contiguous(), dY[rows].contiguous()
    # global amax: MAX over the ranks' local amax (plain and after the RHT)
    loc = torch.tensor([O.amax(Xs), O.amax_rht(Xs), O.amax(dYs), O.amax_rht(dYs)], dtype=torch.float32)
    dist.all_reduce(loc, op=dist.ReduceOp.MAX)
    ax, axr, ag, agr = (float(v) for v in loc)
    cx, sx = O.quantize_row(Xs, ax)
    cxc, sxc = O.quantize_col(Xs, axr, rht=True)
    cgc, sgc = O.quantize_col(dYs, agr, rht=True)
    gs = lambda a: float(O.global_scales(a)[1])
    # partial wgrad over this rank's tokens, then the all-reduce of FP64 dW
    dW, _ = O.gemm(cgc, sgc, gs(agr), cxc, sxc, gs(axr))
    dWt = torch.from_numpy(dW)
    dist.all_reduce(dWt, op=dist.ReduceOp.SUM)
    slowest = bench.max_over_ranks(1.0 + rank, torch.device("cpu"), WORLD)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), ax=ax, axr=axr, ag=ag, agr=agr, cx=cx, sx=sx, cxc=cxc,
             sxc=sxc, dW=dWt.numpy(), slowest=slowest)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_data_parallel_matches_single_process(tmp_path):
    import oracle as O

    mp.start_processes(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, start_method="spawn")
    r = [np.load(tmp_path / f"rank{k}.npz") for k in range(WORLD)]
    X, dY = _inputs()
    ax, axr, ag, agr = O.amax(X), O.amax_rht(X), O.amax(dY), O.amax_rht(dY)
    for k in range(WORLD):
        assert (float(r[k]["ax"]), float(r[k]["axr"]), float(r[k]["ag"]), float(r[k]["agr"])) == (ax, axr, ag, agr)
        assert float(r[k]["slowest"]) == float(WORLD)
    # row copy: ranks hold consecutive row slices
    cx, sx = O.quantize_row(X, ax)
    assert np.array_equal(np.concatenate([r[k]["cx"] for k in range(WORLD)]), cx)
    assert np.array_equal(np.concatenate([r[k]["sx"] for k in range(WORLD)]), sx)
    # column copy (RHT along tokens): ranks hold consecutive slices of the K axis
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    assert np.array_equal(np.concatenate([r[k]["cxc"] for k in range(WORLD)], axis=1), cxc)
    assert np.array_equal(np.concatenate([r[k]["sxc"] for k in range(WORLD)], axis=1), sxc)
    # all-reduced partial wgrad == full-batch wgrad (FP64 sums, up to reassociation)
    cgc, sgc = O.quantize_col(dY, agr, rht=True)
    gs = lambda a: float(O.global_scales(a)[1])
    dW, absum = O.gemm(cgc, sgc, gs(agr), cxc, sxc, gs(axr))
    for k in range(WORLD):
        assert np.all(np.abs(r[k]["dW"] - dW) <= 1e-12 * absum + 1e-300)
