"""Benchmark of the NVFP4 quantized linear layer on B200.

One step = one full pass of the hot path over one batch, through the
data-parallel linear layer (nvfp4_bit_microscaled_b200.dp): forward (amax and
RHT amax of X, X row copy and RHT column copy from one read of X, W amax, W 2D
quantize, fprop GEMM) and backward (amax and RHT amax of dY, dY row quantize with
SR, dgrad GEMM, dY column quantize with RHT + SR, wgrad GEMM), with the
all-reduces of the amaxes (MAX) and of dW (SUM) when there is more than one
rank.  Inputs are seeded synthetic BF16 tensors resident in HBM.

The headline workload is the largest configuration, "large outlier-heavy":
T = 32768 tokens, 8192 -> 8192, X Student-t(3), W N(0, 0.02) with 0.01% of
its entries x50, dY N(0, 1e-3); its three GEMMs are 32768x8192x8192,
32768x8192x8192 and 8192x8192x32768.  The "full" workload (T = 16384,
hidden 5120 -> FFN 20480, a 12B hybrid Mamba-Transformer's up-projection) is
timed the same way and reported in its own object.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank holds T tokens of an N*T-token batch (weak
scaling) and runs the data-parallel step over NCCL; rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain C reference) on the host cores
on a bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_bit_microscaled_b200 import api, dp, synth  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS (% dense FP4 peak); quantize GB/s (% HBM peak)"
WORKLOADS = {
    "large": dict(name="large", T=32768, Cin=8192, Cout=8192, seed=3, sr_seed=3,
                  desc="large outlier-heavy linear fwd+bwd: T=32768, Cin=8192, Cout=8192 (X Student-t(3), "
                       "W N(0,0.02) with 0.01% entries x50, dY N(0,1e-3))"),
    "full": dict(name="full", T=16384, Cin=5120, Cout=20480, seed=2, sr_seed=2,
                 desc="full linear fwd+bwd: T=16384, Cin=5120, Cout=20480 (FFN up-projection of a 12B hybrid "
                      "Mamba-Transformer; X N(0,1) with 0.1% outlier channels x100, W N(0,0.02), "
                      "dY N(0,1e-3) x per-row lognormal)"),
}
HEADLINE = "large"
WORKLOAD = WORKLOADS[HEADLINE]
DENSE_FP4_DATASHEET_TFLOPS = 9000.0
FP4_PER_BF16 = 4.0           # nominal dense FP4 : BF16 tensor ratio (9 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_PROFILE = os.path.join("profiles", "gemm_traffic.json")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def fp4_peak(peaks, src):
    """Dense FP4 roofline: 4 x the burst BF16 GEMM rate (the kernels are timed
    in a sub-second region, where the part runs at its burst clock)."""
    v = FP4_PER_BF16 * peaks["bf16_tflops"]
    return v, f"{src}: 4 x bf16_tflops burst ({peaks['bf16_tflops']}) (nominal dense FP4:BF16 = 9:2.25)"


def gemm_profile():
    """The committed ncu figures of the headline fprop GEMM (DRAM bytes per
    launch, tensor-pipe activity), or None when gemm.cu has changed since
    they were taken (checked by the source hash stored with them)."""
    path = os.path.join(ROOT, GEMM_PROFILE)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        prof = json.load(f)
    src = open(os.path.join(ROOT, "nvfp4_bit_microscaled_b200", "csrc", "gemm.cu"), "rb").read()
    if hashlib.sha256(src).hexdigest() != prof.get("gemm_source_sha256"):
        return None
    return prof


class ClockSampler:
    """SM clocks and throttle reasons sampled during the timed region: NVML from a
    thread every few milliseconds (the timed region can be a fraction of a
    second), else nvidia-smi at its 200 ms floor.  Reads only; sets nothing."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4))
    SMI_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device, enabled=True, period_s=0.005):
        self.device = device              # torch CUDA device index
        self.enabled = enabled
        self.period = period_s
        self.samples = []                 # (time, sm MHz, max sm MHz, set of reason names)
        self.source = None
        self.t0 = self.t1 = None
        self.proc = self.thread = None
        self.nvml = None                  # (module, handle) once NVML answers

    # A timed region of a few tens of milliseconds can pass before the sampling
    # thread gets to run, so the region's two edges are also sampled from the
    # calling thread (NVML only): the first just after the start mark, the
    # last just before the end mark.
    def mark_start(self):
        self.t0 = time.time()
        self._sample_now()

    def mark_end(self):
        self._sample_now()
        self.t1 = time.time()

    def _sample_now(self):
        if self.nvml is None:
            return
        nv, h = self.nvml
        try:
            self._nvml_sample(nv, h)
        except Exception:
            pass

    # -- NVML
    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.device)
        if all(hasattr(p, k) for k in ("pci_domain_id", "pci_bus_id", "pci_device_id")):
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[self.device]) if vis else self.device
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _nvml_sample(self, nv, h):
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        bits = [(n, getattr(nv, attr, v)) for n, attr, v in self.REASONS]
        clk_max = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        clk = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        r = reasons_fn(h)
        self.samples.append((time.time(), float(clk), float(clk_max), {n for n, b in bits if r & b}))

    def _nvml_loop(self, nv, h, stop):
        while True:   # a sample first, then every period until stopped
            try:
                self._nvml_sample(nv, h)
            except Exception:
                pass
            if stop.wait(self.period):
                return

    # -- nvidia-smi
    def _smi_start(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = vis.split(",")[self.device] if vis else str(self.device)
        self.path = os.path.join(tempfile.gettempdir(), f"nvfp4_bench_clocks_{os.getpid()}_{self.device}.csv")
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen(
            ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
             "-i", idx], stdout=self.f, stderr=subprocess.DEVNULL)
        time.sleep(1.0)          # let the sampler start before the timed region

    def _smi_read(self):
        import datetime
        names = [n for n, _, _ in self.REASONS]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    clk, clk_max = float(parts[2]), float(parts[3])
                except ValueError:
                    continue
                self.samples.append((ts, clk, clk_max, {n for n, v in zip(names, parts[6:10])
                                                        if v.lower() == "active"}))
        try:
            os.remove(self.path)
        except OSError:
            pass

    def __enter__(self):
        if not self.enabled:
            return self
        try:
            nv, h = self._nvml_handle()
            self.nvml = (nv, h)
            import threading
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, self.stop), daemon=True)
            self.thread.start()
            self.source = f"nvml every {self.period * 1e3:g} ms"
            return self
        except Exception:
            self.thread = None
        try:
            self._smi_start()
            self.source = "nvidia-smi every 200 ms"
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()
            self._smi_read()

    def summary(self):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        lo, hi = self.t0, self.t1
        inside = [x for x in self.samples if (lo is None or x[0] >= lo) and (hi is None or x[0] <= hi)]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "source": self.source}
        reasons = set().union(*(x[3] for x in inside))
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": max(x[2] for x in inside),
                "reasons": sorted(reasons), "samples": len(inside), "source": self.source}


def max_over_ranks(value, device, world):
    """Max of a per-rank float over all ranks (device timing is reported as the
    slowest rank's)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t[0])


# --------------------------------------------------------------------------- our arm
class EventTimer:
    """timer(kind, fn) for DataParallelLinear: CUDA events around every call on
    the current stream, so per-kernel durations come from inside the timed region."""

    def __init__(self):
        self.record = False
        self.events = []          # (kind, start, end)

    def __call__(self, kind, fn):
        if not self.record:
            return fn()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        out = fn()
        e.record()
        self.events.append((kind, s, e))
        return out


class AloneTimer:
    """timer(kind, fn) that times each library call alone, after the step's
    timed region: the device is idle before every launch (so no kernel of the
    other stream runs beside it), L2 is flushed with a 256 MB write, and the
    call is launched once untimed, then `reps` times timed; collectives run
    once, untimed.

    The device would reach the start event as soon as the flush ends, while
    the host may still be inside the call (argument marshalling, the launch):
    that gap would be timed as the kernel's.  A device-side wait of `hold_cycles`
    after the flush keeps the device busy until the call is enqueued, as it is
    in the back-to-back step."""

    def __init__(self, device, reps=5, hold_cycles=1_000_000):
        self.reps = reps
        self.hold_cycles = hold_cycles
        self.ms = {}
        self.scratch = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def __call__(self, kind, fn):
        if kind.startswith("allreduce"):
            return fn()
        out = fn()   # untimed: the call's first-use work (an output allocation, a descriptor) is done here
        times = []
        for _ in range(self.reps):
            out = None   # the previous output goes back to the allocator's cache, so the call reuses it
            torch.cuda.synchronize()
            self.scratch.fill_(1)
            if self.hold_cycles:
                torch.cuda._sleep(self.hold_cycles)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            out = fn()
            e.record()
            torch.cuda.synchronize()
            times.append(s.elapsed_time(e))
        self.ms.setdefault(kind, []).append(sum(times) / len(times))
        return out


KERNELS_PER_STEP = 10  # 3 amax + 4 quantize + 3 GEMM kernels (no scale padding at these shapes)
QUANT_KINDS = ("quant_rowcol_rht", "quant_2d", "quant_row_sr", "quant_col_rht_sr")


def kernel_bytes(T, Ci, Co):
    """Algorithmic HBM bytes per step of each kernel kind (reads + writes of the data the op must touch)."""
    q = lambda r, c: r * c / 2 + r * c / 16          # packed codes + one scale byte per 16
    return {
        "amax": 2.0 * Ci * Co,
        "amax_both": 2.0 * (T * Ci + T * Co),
        "quant_rowcol_rht": 2.0 * T * Ci + 2 * q(T, Ci),      # X read once, row copy + RHT column copy
        "quant_2d": 2.0 * Co * Ci + 2 * q(Co, Ci),
        "quant_row_sr": 2.0 * T * Co + q(T, Co),
        "quant_col_rht_sr": 2.0 * T * Co + q(T, Co),
    }


def gemm_flops(T, Ci, Co):
    return {"gemm_fprop": 2.0 * T * Co * Ci, "gemm_dgrad": 2.0 * T * Ci * Co, "gemm_wgrad": 2.0 * Co * Ci * T}


def make_inputs(wl, rank, device):
    """This rank's T tokens of the batch (its own seed) and the replicated W."""
    name, T, Ci, Co = wl["name"], wl["T"], wl["Cin"], wl["Cout"]
    seed = wl["seed"] + 1000 * rank
    if name == "large":
        X = synth.heavy_activations(T, Ci, seed, device=device)
        W = synth.weights(Co, Ci, wl["seed"], device=device, outlier_frac=1e-4, outlier_scale=50.0)
        dY = synth.gradients(T, Co, seed, device=device, row_lognormal=False)
    else:
        X = synth.activations(T, Ci, seed, device=device)
        W = synth.weights(Co, Ci, wl["seed"], device=device)
        dY = synth.gradients(T, Co, seed, device=device)
    return X, W, dY


def time_step(wl, args, rank, world, device, clocks=True):
    """W warm-up steps, then K timed steps of the data-parallel layer between
    barriers; device time from CUDA events, max over ranks."""
    T, Ci, Co = wl["T"], wl["Cin"], wl["Cout"]
    X, W, dY = make_inputs(wl, rank, device)
    timer = EventTimer()
    layer = dp.DataParallelLinear(T, Ci, Co, device, timer=timer)
    Y = torch.empty(T, Co, dtype=torch.bfloat16, device=device)
    dX = torch.empty(T, Ci, dtype=torch.bfloat16, device=device)
    dW = torch.empty(Co, Ci, dtype=torch.float32, device=device)

    def step():
        layer.forward(X, W, Y=Y)
        layer.backward(dY, wl["sr_seed"], dX=dX, dW=dW)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    api.read_device_error(clear=True)

    timer.record = True
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device(), enabled=clocks) as clk:
        clk.mark_start()
        start.record()
        for _ in range(args.steps):
            step()
        end.record()
        torch.cuda.synchronize()
        clk.mark_end()
    if world > 1:
        torch.distributed.barrier()
    ms_total = start.elapsed_time(end)
    err = api.read_device_error(clear=True)
    if err:
        raise RuntimeError(f"device error word {err} after the timed region")

    # every kernel once more, alone (outside the timed region; the step above is the number)
    alone = AloneTimer(device)
    layer.timer = alone
    step()
    torch.cuda.synchronize()
    layer.timer = timer
    err = api.read_device_error(clear=True)
    if err:
        raise RuntimeError(f"device error word {err} after the isolated timings")

    per_kind = {}
    for kind, s, e in timer.events:
        per_kind.setdefault(kind, []).append(s.elapsed_time(e))
    avg_ms = {k: sum(v) / len(v) for k, v in per_kind.items()}
    total_ms = {k: sum(v) / args.steps for k, v in per_kind.items()}
    ms_step = max_over_ranks(ms_total, device, world) / args.steps
    flops_step = 3 * 2.0 * T * Ci * Co

    peaks, peak_src = load_peaks()
    fpeak, fpeak_src = fp4_peak(peaks, peak_src)
    hbm = peaks["hbm_gbs"]
    gf = gemm_flops(T, Ci, Co)
    kb = kernel_bytes(T, Ci, Co)
    g_ms = sum(total_ms[k] for k in gf)
    q_ms = sum(total_ms[k] for k in QUANT_KINDS)
    a_ms = total_ms["amax"] + total_ms["amax_both"]
    kernels = {}
    for k in avg_ms:
        n = len(per_kind[k]) // args.steps
        entry = {"ms_per_launch": round(avg_ms[k], 4), "launches_per_step": n}
        if k in gf:
            entry["tflops"] = round(gf[k] / (avg_ms[k] * 1e-3) / 1e12, 1)
            entry["frac_fp4_peak"] = round(entry["tflops"] / fpeak, 4)
        elif k in kb:
            entry["gbs"] = round(kb[k] / n / (avg_ms[k] * 1e-3) / 1e9, 1)
            entry["frac_hbm"] = round(entry["gbs"] / hbm, 4)
        kernels[k] = entry
    kernels_alone = {}
    for k, v in alone.ms.items():
        ms = sum(v) / len(v)
        entry = {"ms_per_launch": round(ms, 4)}
        if k in gf:
            entry["tflops"] = round(gf[k] / (ms * 1e-3) / 1e12, 1)
            entry["frac_fp4_peak"] = round(entry["tflops"] / fpeak, 4)
        elif k in kb:
            entry["gbs"] = round(kb[k] / len(v) / (ms * 1e-3) / 1e9, 1)
            entry["frac_hbm"] = round(entry["gbs"] / hbm, 4)
        kernels_alone[k] = entry
    return {
        "workload": wl["desc"],
        "ms_per_step": round(ms_step, 4),
        "value": round(flops_step * world / (ms_step * 1e-3) / 1e12, 2),
        "gemm": {
            "tflops_gemm_only": round(sum(gf.values()) / (g_ms * 1e-3) / 1e12, 1),
            "frac_fp4_peak": round(sum(gf.values()) / (g_ms * 1e-3) / 1e12 / fpeak, 4),
            "frac_fp4_datasheet_9pf": round(sum(gf.values()) / (g_ms * 1e-3) / 1e12 / DENSE_FP4_DATASHEET_TFLOPS, 4),
            "share_of_step": round(g_ms / ms_step, 3),
        },
        "quantize": {
            "gbs": round(sum(kb[k] for k in QUANT_KINDS) / (q_ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(sum(kb[k] for k in QUANT_KINDS) / (q_ms * 1e-3) / 1e9 / hbm, 4),
            "amax_gbs": round((kb["amax"] + kb["amax_both"]) / (a_ms * 1e-3) / 1e9, 1),
            "amax_frac_hbm": round((kb["amax"] + kb["amax_both"]) / (a_ms * 1e-3) / 1e9 / hbm, 4),
            "share_of_step": round((q_ms + a_ms) / ms_step, 3),
        },
        "kernels": kernels,
        "streams": ("W's amax and 2D quantize run on a second stream beside X's amax and ROWCOL quantize; "
                    "quant_row_sr runs beside gemm_wgrad: per-kernel times are taken on each kernel's own "
                    "stream, so overlapping shares can sum above 1"),
        "kernels_alone": kernels_alone,
        "kernels_alone_note": ("each call once more after the timed region, alone on an idle device, L2 "
                               "flushed before each of 5 launches, each enqueued behind a short device-side "
                               "wait so that the host's launch time is not timed: the kernel's own rate, "
                               "without the second stream's overlap"),
        "_fprop": (gf["gemm_fprop"], avg_ms["gemm_fprop"], fpeak, fpeak_src),
        "_clocks": clk.summary(),
        "_tensors": (X, W, dY),
    }


def run_ours(args, rank, world, device):
    wl = WORKLOAD
    T, Ci, Co = wl["T"], wl["Cin"], wl["Cout"]
    head = time_step(wl, args, rank, world, device)
    flops, fprop_ms, fpeak, fpeak_src = head.pop("_fprop")
    achieved = flops / (fprop_ms * 1e-3) / 1e12
    prof = gemm_profile()
    result = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, fp32 accumulate)",
        "data": "synthetic (seeded; X Student-t(3), W N(0,0.02) with 0.01% entries x50, dY N(0,1e-3))",
        "config": workload_config(world),
        "gemm": head["gemm"],
        "quantize": head["quantize"],
        "kernels": head["kernels"],
        "streams": head["streams"],
        "kernels_alone": head["kernels_alone"],
        "kernels_alone_note": head["kernels_alone_note"],
        "roofline": {
            "kernel": f"gemm_fp4_pair_kernel<false, false> (fprop, M={T} N={Co} K={Ci}, BF16 out)",
            "bound": "tensor",
            "achieved": round(achieved, 1),
            "peak": round(fpeak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / fpeak, 4),
            "peak_source": fpeak_src,
            "frac_of_datasheet_9pf": round(achieved / DENSE_FP4_DATASHEET_TFLOPS, 4),
            "traffic": prof["traffic_bytes_per_launch"] if prof else None,
            "tensor_pipe_pct": prof.get("tensor_pipe_pct") if prof else None,
            "algorithmic_bytes": (T + Co) * Ci * 0.5625 + T * Co * 2,
        },
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": head["_clocks"],
    }
    if world > 1:
        result["nccl_ranks"] = torch.distributed.get_world_size()
    tensors = head.pop("_tensors")
    del tensors
    torch.cuda.empty_cache()
    other = dict(WORKLOADS["full"])
    full = time_step(other, args, rank, world, device, clocks=False)
    full.pop("_fprop"), full.pop("_clocks"), full.pop("_tensors")
    result["full_workload"] = full
    return result


def run_e2e(args, rank, world, device):
    """Same metric end to end through the public API with host buffers: every
    step copies its X, W, dY from pinned host memory to the device and its Y,
    dX, dW back to pinned host memory, inside the timed region.  One GPU runs
    nvfp4_linear_fwd / nvfp4_linear_bwd (the C ABI's linear calls); several
    run the data-parallel layer.  Copies run on their own streams and are
    pipelined across steps (inputs of step i+1 and outputs of step i-1 move
    while step i computes), with two device buffer sets; the data dependencies
    are kept by events."""
    wl = WORKLOAD
    T, Ci, Co = wl["T"], wl["Cin"], wl["Cout"]
    steps = max(2, min(args.steps, 24))   # enough that filling and draining the copy pipeline is a small part
    X, W, dY = make_inputs(wl, rank, device)
    hin = [tuple(t.cpu().pin_memory() for t in (X, W, dY)) for _ in range(2)]
    del X, W, dY
    hout = [(torch.empty(T, Co, dtype=torch.bfloat16).pin_memory(),
             torch.empty(T, Ci, dtype=torch.bfloat16).pin_memory(),
             torch.empty(Co, Ci, dtype=torch.float32).pin_memory()) for _ in range(2)]
    din = [tuple(torch.empty_like(h, device=device) for h in hin[0]) for _ in range(2)]
    dout = [tuple(torch.empty_like(h, device=device) for h in hout[0]) for _ in range(2)]
    if world == 1:
        ws = [api.LinearWorkspace(T, Ci, Co, device) for _ in range(2)]

        def compute(b):
            Xd, Wd, Gd = din[b]
            Y, gX, gW = dout[b]
            api.linear_fwd(Xd, Wd, ws[b], Y=Y)
            api.linear_bwd(Gd, ws[b], wl["sr_seed"], dX=gX, dW=gW)
    else:
        layers = [dp.DataParallelLinear(T, Ci, Co, device) for _ in range(2)]

        def compute(b):
            Xd, Wd, Gd = din[b]
            Y, gX, gW = dout[b]
            layers[b].forward(Xd, Wd, Y=Y)
            layers[b].backward(Gd, wl["sr_seed"], dX=gX, dW=gW)
    compute_s, h2d, d2h = torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        loaded = [None, None]      # event: inputs of buffer b on the device
        computed = [None, None]    # event: outputs of buffer b ready
        drained = [None, None]     # event: outputs of buffer b copied out (buffer b reusable)
        consumed = [None, None]    # event: inputs of buffer b no longer needed

        def load(i):
            b = i % 2
            with torch.cuda.stream(h2d):
                if consumed[b] is not None:
                    h2d.wait_event(consumed[b])
                for d, h in zip(din[b], hin[b]):
                    d.copy_(h, non_blocking=True)
                loaded[b] = torch.cuda.Event()
                loaded[b].record(h2d)
        load(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                load(i + 1)
            compute_s.wait_event(loaded[b])
            if drained[b] is not None:
                compute_s.wait_event(drained[b])
            compute(b)
            consumed[b] = torch.cuda.Event()
            consumed[b].record(compute_s)
            computed[b] = torch.cuda.Event()
            computed[b].record(compute_s)
            with torch.cuda.stream(d2h):
                d2h.wait_event(computed[b])
                for h, d in zip(hout[b], dout[b]):
                    h.copy_(d, non_blocking=True)
                drained[b] = torch.cuda.Event()
                drained[b].record(d2h)
        compute_s.wait_event(drained[(n - 1) % 2])
        if n > 1:
            compute_s.wait_event(drained[(n - 2) % 2])

    run(2)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(compute_s)
    h2d.wait_event(s)
    d2h.wait_event(s)
    run(steps)
    e.record(compute_s)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), device, world)
    ms_step = ms / steps
    flops = 3 * 2.0 * T * Ci * Co
    h2d_b = sum(t.numel() * t.element_size() for t in hin[0])
    d2h_b = sum(t.numel() * t.element_size() for t in hout[0])
    return {"value": round(flops * world / (ms_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b, "ms_per_step": round(ms_step, 3),
            "steps": steps, "api": "nvfp4_linear_fwd/_bwd" if world == 1 else "DataParallelLinear (NCCL)",
            "pipelined": "H2D of step i+1 and D2H of step i-1 overlap step i (copy streams)"}


# --------------------------------------------------------------------------- reference arm
def oracle_sample(seconds_target=15.0):
    """The CPU oracle on a bounded sample of the headline workload: the six
    quantizations of a 64-token slice of the batch and W's first 256 rows, and
    FP64 GEMM entries sampled from fprop and wgrad.  Returns (TFLOP/s of GEMM
    work, cores, description, seconds)."""
    import numpy as np

    import oracle as O

    wl = WORKLOAD
    Ci, Co = wl["Cin"], wl["Cout"]
    Ts = 64
    X = synth.heavy_activations(Ts, Ci, wl["seed"])
    W = synth.weights(256, Ci, wl["seed"], outlier_frac=1e-4, outlier_scale=50.0)
    dY = synth.gradients(Ts, Co, wl["seed"], row_lognormal=False)
    rng = np.random.default_rng(0)
    flops = 0.0
    t0 = time.perf_counter()
    ax, aw, ag = O.amax(X), O.amax(W), O.amax(dY)
    axr, agr = O.amax_rht(X), O.amax_rht(dY)
    cx, sx = O.quantize_row(X, ax)
    cw, tw = O.quantize_2d(W, aw)
    (cwr, swr), (cwc, swc) = O.expand_2d(cw, tw)
    cxc, sxc = O.quantize_col(X, axr, rht=True)
    cg, sg = O.quantize_row(dY, ag, sr=True, seed=wl["sr_seed"])
    cgc, sgc = O.quantize_col(dY, agr, rht=True, sr=True, seed=wl["sr_seed"])
    gs = lambda a: float(O.global_scales(a)[1])
    n = 512
    while True:
        p1 = np.stack([rng.integers(0, Ts, n), rng.integers(0, 256, n)], 1)
        O.gemm(cx, sx, gs(ax), cwr, swr, gs(aw), pairs=p1)                 # fprop entries, K = Cin
        p3 = np.stack([rng.integers(0, Co, n), rng.integers(0, Ci, n)], 1)
        O.gemm(cgc, sgc, gs(agr), cxc, sxc, gs(axr), pairs=p3)             # wgrad entries, K = Ts
        flops += 2.0 * n * Ci + 2.0 * n * Ts
        if time.perf_counter() - t0 > seconds_target:
            break
    dt = time.perf_counter() - t0
    desc = (f"oracle (plain C, OpenMP) on host cores: amax/quantize of a {Ts}-token slice of X and dY and of "
            f"W[:256] of the large workload, then FP64 GEMM entries sampled from fprop (K={Ci}) and wgrad "
            f"(K={Ts}) for ~{seconds_target:.0f}s")
    return flops / dt / 1e12, O.num_threads(), desc, dt


def workload_config(world):
    """The config object both arms print: the headline workload."""
    T, Ci, Co = WORKLOAD["T"], WORKLOAD["Cin"], WORKLOAD["Cout"]
    return {
        "workload": WORKLOAD["desc"] + "; 3 GEMMs, 3 amax, 4 quantize kernels per step",
        "T": T, "Cin": Ci, "Cout": Co,
        "parallelism": f"dp{world}" + (" (NCCL all-reduce of amaxes and dW)" if world > 1 else ""),
        "l2": f"inputs larger than L2 (X {2 * T * Ci / 1e6:.0f} MB, W {2 * Co * Ci / 1e6:.0f} MB, "
              f"dY {2 * T * Co / 1e6:.0f} MB; L2 126 MB): no flush needed",
    }


def run_reference(args, rank, world):
    if rank != 0:
        return None
    steps = []
    # the whole run (warm-up and timed steps) stays near a minute whatever K and W are
    per = max(0.2, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(per)
    for _ in range(args.steps):
        v, cores, desc, dt = oracle_sample(per)
        steps.append((v, dt))
    value = statistics.mean(v for v, _ in steps)
    ms = statistics.mean(dt for _, dt in steps) * 1e3
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64 GEMM on fp32-quantized operands",
        "data": "synthetic (seeded)",
        "config": workload_config(world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


CASES = ("gemm", "gemm_amax", "amax", "amax_rht", "amax_both", "quant_row", "quant_row_sr", "quant_2d", "quant_col_rht",
         "quant_col_rht_sr", "quant_rowcol_rht", "mx_gemm", "mx_quant_row")


def _event_ms(fn, reps):
    """Average device time of fn() over reps launches on the current stream."""
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / reps


def measure_mxfp4(X, W, reps=20):
    """The MXFP4 comparison format on the fprop operands of the workload:
    1x32 UE8M0 quantization of X and W, then Y = X W^T (BF16 out) on the
    block-32 CTA-pair kernel.  Timed on its own, after the step timing."""
    T, Ci = X.shape
    Co = W.shape[0]
    qx, qw = api.mx_quantize(X), api.mx_quantize(W)
    Y = torch.empty(T, Co, dtype=torch.bfloat16, device=X.device)
    for _ in range(3):
        api.mx_quantize(X, out=qx)
        api.mx_gemm(qx, qw, api.OUT_BF16, out=Y)
    torch.cuda.synchronize()
    q_ms = _event_ms(lambda: api.mx_quantize(X, out=qx), reps)
    g_ms = _event_ms(lambda: api.mx_gemm(qx, qw, api.OUT_BF16, out=Y), reps)
    peaks, src = load_peaks()
    fpeak, _ = fp4_peak(peaks, src)
    q_bytes = T * Ci * (2 + 0.5 + 1 / 32)
    tflops = 2.0 * T * Co * Ci / (g_ms * 1e-3) / 1e12
    gbs = q_bytes / (q_ms * 1e-3) / 1e9
    return {"gemm_fprop": {"ms_per_launch": round(g_ms, 4), "tflops": round(tflops, 1),
                           "frac_fp4_peak": round(tflops / fpeak, 4)},
            "quant_row_x": {"ms_per_launch": round(q_ms, 4), "gbs": round(gbs, 1),
                            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)},
            "note": "comparison format (1x32 blocks, UE8M0 scales, no tensor scale); not part of the step"}


def measure_epilogue_amax(X, W, rounds=4, reps=8):
    """The fprop GEMM of the workload with the amax of Y reduced in its
    epilogue (nvfp4_gemm_amax), against the plain GEMM followed by a separate
    amax pass over Y: what quantizing Y for a following GEMM saves.  The three
    are timed in turn over several rounds (medians), after the step timing."""
    T = X.shape[0]
    Co = W.shape[0]
    ax, aw = api.amax(X), api.amax(W)
    xr, _ = api.quantize(X, api.ROW, ax)
    wr, _ = api.quantize(W, api.TWO_D, aw, col_out=False)
    Y = torch.empty(T, Co, dtype=torch.bfloat16, device=X.device)
    a1 = torch.empty(1, dtype=torch.float32, device=X.device)
    a2 = torch.empty(1, dtype=torch.float32, device=X.device)
    plain = lambda: api.gemm(xr, wr, api.OUT_BF16, out=Y)
    fused = lambda: api.gemm_amax(xr, wr, api.OUT_BF16, out=Y, amax_out=a1)
    sep = lambda: api.amax(Y, out=a2)
    for _ in range(3):
        plain(), fused(), sep()
    torch.cuda.synchronize()
    g, f, a = [], [], []
    for _ in range(rounds):
        g.append(_event_ms(plain, reps))
        f.append(_event_ms(fused, reps))
        a.append(_event_ms(sep, reps))
    med = lambda v: sorted(v)[len(v) // 2]
    g_ms, f_ms, a_ms = med(g), med(f), med(a)
    assert float(a1.cpu()[0]) == float(a2.cpu()[0]), "epilogue amax differs from the amax pass"
    return {"gemm_ms": round(g_ms, 4), "gemm_amax_ms": round(f_ms, 4), "amax_pass_ms": round(a_ms, 4),
            "saved_ms": round(g_ms + a_ms - f_ms, 4),
            "note": "fprop Y = X W^T (BF16) with max|Y| from the epilogue vs GEMM + amax pass over Y; "
                    "not part of the step"}


def run_case(args):
    """One kernel alone on a given shape (ncu captures, launch-shape sweeps).
    gemm: --shape M,N,K (A activations, B weights, BF16 out); the others:
    --shape R,C of the BF16 input.  Prints one JSON line."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    shape = [int(v) for v in args.shape.split(",")]
    from nvfp4_bit_microscaled_b200 import build as libbuild
    libbuild.build()
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    if args.case == "mx_gemm":
        M, N, K = shape
        qa = api.mx_quantize(synth.activations(M, K, 5, device=dev))
        qb = api.mx_quantize(synth.weights(N, K, 5, device=dev))
        D = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        fn = lambda: api.mx_gemm(qa, qb, api.OUT_BF16, out=D)
        work, unit = 2.0 * M * N * K, "TFLOP/s"
    elif args.case == "mx_quant_row":
        R, C = shape
        x = synth.activations(R, C, 5, device=dev)
        q = api.mx_quantize(x)
        fn, work, unit = (lambda: api.mx_quantize(x, out=q)), R * C * (2 + 0.5 + 1 / 32), "GB/s"
    elif args.case in ("gemm", "gemm_amax"):
        M, N, K = shape
        a_in, b_in = synth.activations(M, K, 5, device=dev), synth.weights(N, K, 5, device=dev)
        qa, _ = api.quantize(a_in, api.ROW, api.amax(a_in))
        qb, _ = api.quantize(b_in, api.ROW, api.amax(b_in))
        f32 = args.out == "f32"
        D = torch.empty(M, N, dtype=torch.float32 if f32 else torch.bfloat16, device=dev)
        od = api.OUT_F32 if f32 else api.OUT_BF16
        if args.case == "gemm":
            fn = lambda: api.gemm(qa, qb, od, out=D)
        else:
            fn = lambda: api.gemm_amax(qa, qb, od, out=D, amax_out=amax)
        work, unit = 2.0 * M * N * K, "TFLOP/s"
    else:
        R, C = shape
        x = synth.gradients(R, C, 5, device=dev) if "sr" in args.case else synth.activations(R, C, 5, device=dev)
        api.amax(x, rht="rht" in args.case, out=amax)
        qbytes = R * C / 2 + R * C / 16
        if args.case == "amax":
            fn, work = (lambda: api.amax(x, out=amax)), 2.0 * R * C
        elif args.case == "amax_rht":
            fn, work = (lambda: api.amax(x, rht=True, out=amax)), 2.0 * R * C
        elif args.case == "amax_both":
            amax2 = torch.zeros(2, dtype=torch.float32, device=dev)
            fn, work = (lambda: api.amax(x, rht=2, out=amax2)), 2.0 * R * C
        elif args.case in ("quant_row", "quant_row_sr"):
            q = api.empty_qtensor(R, C, dev)
            sr = args.case.endswith("sr")
            fn, work = (lambda: api.quantize(x, api.ROW, amax, sr=sr, seed=1, row_out=q)), 2.0 * R * C + qbytes
        elif args.case == "quant_rowcol_rht":
            a2 = torch.zeros(2, dtype=torch.float32, device=dev)
            api.amax(x, rht=2, out=a2)
            qr, qc = api.empty_qtensor(R, C, dev), api.empty_qtensor(C, R, dev)
            fn, work = (lambda: api.quantize(x, api.ROWCOL, a2, rht=True, row_out=qr, col_out=qc)), \
                2.0 * R * C + 2 * qbytes
        elif args.case == "quant_2d":
            qr, qc = api.empty_qtensor(R, C, dev), api.empty_qtensor(C, R, dev)
            fn, work = (lambda: api.quantize(x, api.TWO_D, amax, row_out=qr, col_out=qc)), 2.0 * R * C + 2 * qbytes
        else:
            q = api.empty_qtensor(C, R, dev)
            sr = args.case.endswith("sr")
            fn, work = (lambda: api.quantize(x, api.COL, amax, rht=True, sr=sr, seed=1, col_out=q)), \
                2.0 * R * C + qbytes
        unit = "GB/s"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    if args.flush:
        # inputs that fit in L2 would be re-read from it: evict between launches, time each launch alone
        scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for s, e in evs:
            scratch.fill_(1)
            s.record()
            fn()
            e.record()
        torch.cuda.synchronize()
        ms = sum(s.elapsed_time(e) for s, e in evs) / args.steps
    else:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            fn()
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / args.steps
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"case": args.case, "shape": shape, "out": args.out if "gemm" in args.case else None,
                      "flush": bool(args.flush), "ms_per_launch": round(ms, 4), "rate": round(rate, 1),
                      "unit": unit}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=CASES, help="time one kernel alone on --shape")
    ap.add_argument("--shape", default="")
    ap.add_argument("--out", choices=["bf16", "f32"], default="bf16", help="--case gemm: output type")
    ap.add_argument("--flush", action="store_true",
                    help="--case: write a 256 MiB buffer (twice L2) before each launch and time launches one by one")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.case:
        run_case(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if world > 1:
            import datetime
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    from nvfp4_bit_microscaled_b200 import build as libbuild
    libbuild.build()

    result = run_ours(args, rank, world, device)
    if not args.no_e2e:
        torch.cuda.empty_cache()
        result["e2e"] = run_e2e(args, rank, world, device)
    torch.cuda.empty_cache()
    X, W, _ = make_inputs(WORKLOAD, rank, device)
    result["mxfp4"] = measure_mxfp4(X, W)
    result["epilogue_amax"] = measure_epilogue_amax(X, W)
    del X, W
    if rank == 0 and not args.no_cpu_baseline:
        v, cores, desc, dt = oracle_sample(12.0)
        result["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
