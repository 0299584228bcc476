"""The linear layer's second stream: nvfp4_linear_fwd/_bwd and the
data-parallel layer run independent branches (W's quantizers in the forward,
the dY row copy next to the wgrad GEMM in the backward) on a stream of their
own, forked from and joined back to the caller's stream.  These tests check
that the results do not depend on that overlap: back-to-back calls with no
host synchronisation, a caller on a non-default stream, and a captured CUDA
graph all give the bytes of calls made one at a time."""
import pytest
import torch

from nvfp4_bit_microscaled_b200 import api, synth
from nvfp4_bit_microscaled_b200.dp import DataParallelLinear
from tests._parity import dev

pytestmark = pytest.mark.gpu

T, CIN, COUT = 512, 640, 384


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


def _steps(n):
    # a different X, W and dY in every step, so a step that read a neighbour's
    # operands would differ
    return [(dev(synth.activations(T, CIN, 300 + i)), dev(synth.weights(COUT, CIN, 400 + i)),
             dev(synth.gradients(T, COUT, 500 + i))) for i in range(n)]


def _one_step(X, W, dY, ws, seed, outs):
    Y, dX, dW = outs
    api.linear_fwd(X, W, ws, Y=Y)
    api.linear_bwd(dY, ws, seed, dX=dX, dW=dW)


def _outs():
    return (torch.empty(T, COUT, dtype=torch.bfloat16, device="cuda"),
            torch.empty(T, CIN, dtype=torch.bfloat16, device="cuda"),
            torch.empty(COUT, CIN, dtype=torch.float32, device="cuda"))


def _serial(steps, seeds=None):
    ws = api.LinearWorkspace(T, CIN, COUT, "cuda")
    ref = []
    for i, (X, W, dY) in enumerate(steps):
        outs = _outs()
        _one_step(X, W, dY, ws, 77 + i if seeds is None else seeds[i], outs)
        torch.cuda.synchronize()
        ref.append(outs)
    return ref


def _assert_same(got, ref):
    for i, (g, r) in enumerate(zip(got, ref)):
        for name, a, b in zip(("Y", "dX", "dW"), g, r):
            assert torch.equal(a, b), f"step {i}: {name} differs from the one-call-at-a-time result"


def test_back_to_back_calls_match_serial_calls():
    steps = _steps(6)
    ref = _serial(steps)
    ws = api.LinearWorkspace(T, CIN, COUT, "cuda")
    got = [_outs() for _ in steps]
    torch.cuda.synchronize()
    for i, (X, W, dY) in enumerate(steps):      # one workspace, no host sync in between
        _one_step(X, W, dY, ws, 77 + i, got[i])
    torch.cuda.synchronize()
    _assert_same(got, ref)


def test_caller_on_a_non_default_stream():
    steps = _steps(3)
    ref = _serial(steps)
    ws = api.LinearWorkspace(T, CIN, COUT, "cuda")
    got = [_outs() for _ in steps]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i, (X, W, dY) in enumerate(steps):
            _one_step(X, W, dY, ws, 77 + i, got[i])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    _assert_same(got, ref)


def test_captured_graph_replays_the_fork_and_join():
    steps = _steps(2)
    ref = _serial(steps, seeds=[77, 77])         # the seed is a kernel argument: fixed in the graph
    ws = api.LinearWorkspace(T, CIN, COUT, "cuda")
    X, W, dY = (t.clone() for t in steps[0])
    outs = _outs()
    _one_step(X, W, dY, ws, 77, outs)           # eager call first: side stream and events exist
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _one_step(X, W, dY, ws, 77, outs)
    for i in (1, 0):
        for dst, src in zip((X, W, dY), steps[i]):
            dst.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        _assert_same([outs], [ref[i]])
    del g


def test_dp_layer_back_to_back_steps_match_serial_steps():
    steps = _steps(4)
    layer = DataParallelLinear(T, CIN, COUT, "cuda")
    ref = []
    for i, (X, W, dY) in enumerate(steps):
        Y = layer.forward(X, W)
        dX, dW = layer.backward(dY, seed=9 + i)
        torch.cuda.synchronize()
        ref.append((Y.clone(), dX.clone(), dW.clone()))
    layer = DataParallelLinear(T, CIN, COUT, "cuda")
    got = []
    for i, (X, W, dY) in enumerate(steps):
        Y = layer.forward(X, W, Y=torch.empty(T, COUT, dtype=torch.bfloat16, device="cuda"))
        dX, dW = layer.backward(dY, seed=9 + i, dX=torch.empty(T, CIN, dtype=torch.bfloat16, device="cuda"),
                                dW=torch.empty(COUT, CIN, dtype=torch.float32, device="cuda"))
        got.append((Y, dX, dW))
    torch.cuda.synchronize()
    _assert_same(got, ref)


def test_two_host_threads_share_the_side_stream():
    # each thread: its own workspace and caller stream; the library's side stream is shared
    import threading
    steps = _steps(4)
    ref = _serial(steps)
    got = [_outs() for _ in steps]
    torch.cuda.synchronize()
    errors = []

    def worker(idx):
        try:
            ws = api.LinearWorkspace(T, CIN, COUT, "cuda")
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for i in idx:
                    X, W, dY = steps[i]
                    _one_step(X, W, dY, ws, 77 + i, got[i])
            s.synchronize()
        except Exception as e:   # reported by the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(idx,)) for idx in ((0, 2), (1, 3))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not errors, errors
    torch.cuda.synchronize()
    _assert_same(got, ref)
