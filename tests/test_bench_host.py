"""Host-side logic of bench.py, CPU only: the clock record that decides whether
a run is kept (samples outside the timed region ignored, throttle reasons
collected, median clock), the GEMM profile figures that are reported only while
the kernel source still matches the ncu capture, the roofline peak, and the
config object both arms print."""
import datetime
import hashlib
import json
import os
import re
import time

import bench


def _line(ts, sm, reasons=("Not Active",) * 4):
    stamp = datetime.datetime.fromtimestamp(ts).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return ", ".join([stamp, "0", str(sm), "1965", "990.0", "0x0000000000000004", *reasons]) + "\n"


def _smi_sampler(tmp_path, lines):
    c = bench.ClockSampler(0)
    c.path = str(tmp_path / "clocks.csv")
    c.source = "nvidia-smi every 200 ms"
    with open(c.path, "w") as f:
        f.writelines(lines)
    c._smi_read()
    return c


def test_clock_summary_keeps_timed_samples_and_reasons(tmp_path):
    t0 = 1_800_000_000.0
    c = _smi_sampler(tmp_path, [
        _line(t0 - 5.0, 600, ("Active",) * 4),                 # before the timed region
        _line(t0 + 1.0, 1700),
        _line(t0 + 2.0, 1650, ("Not Active", "Not Active", "Not Active", "Active")),
        _line(t0 + 3.0, 1750),
        "garbage line\n",
        _line(t0 + 20.0, 300, ("Active",) * 4)])               # after it
    c.t0, c.t1 = t0, t0 + 10.0
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1700 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(c.path)


def test_clock_summary_flags_hardware_slowdown(tmp_path):
    t0 = 1_800_000_000.0
    c = _smi_sampler(tmp_path, [_line(t0 + 1.0, 1200, ("Active", "Not Active", "Active", "Not Active"))])
    c.t0, c.t1 = t0, t0 + 10.0
    assert c.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples(tmp_path):
    c = bench.ClockSampler(0)
    assert c.summary()["reasons"] == ["clock sampling unavailable"]
    c = _smi_sampler(tmp_path, [])
    assert c.summary()["reasons"] == ["no samples"]


class _FakeNvml:
    """Clock queries of a fake NVML: a clock sequence and one reason bit mask."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40

    def __init__(self, clocks, reasons):
        self.clocks, self.reasons, self.calls = list(clocks), reasons, 0

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls += 1
        return self.clocks[min(self.calls - 1, len(self.clocks) - 1)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_nvml_sampler_decodes_reason_bits():
    import threading
    nv = _FakeNvml([1500, 1520, 1480], 0x4 | 0x1)            # power cap (+ the idle bit, not reported)
    c = bench.ClockSampler(0, period_s=0.001)
    c.source = "nvml"
    stop = threading.Event()
    th = threading.Thread(target=c._nvml_loop, args=(nv, None, stop))
    c.mark_start()
    th.start()
    deadline = time.time() + 10.0
    while nv.calls < 5 and time.time() < deadline:
        time.sleep(0.001)
    stop.set()
    th.join()
    c.mark_end()
    s = c.summary()
    assert s["sm_max_mhz"] == 1965 and s["samples"] >= 3
    assert s["reasons"] == ["sw_power_cap"] and s["sm_mhz"] in (1480, 1500, 1520)


def test_short_timed_region_still_gets_its_edge_samples():
    # no sampling thread at all: the start and end marks sample NVML themselves
    nv = _FakeNvml([1900, 1910], 0x4)
    c = bench.ClockSampler(0)
    c.source = "nvml"
    c.nvml = (nv, None)
    c.mark_start()
    c.mark_end()
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1905.0 and s["reasons"] == ["sw_power_cap"]


def test_gemm_profile_is_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    root = tmp_path
    (root / "profiles").mkdir()
    (root / "nvfp4_bit_microscaled_b200" / "csrc").mkdir(parents=True)
    src = b"// kernel source\n"
    (root / "nvfp4_bit_microscaled_b200" / "csrc" / "gemm.cu").write_bytes(src)
    prof = {"traffic_bytes_per_launch": 1234567, "tensor_pipe_pct": 71.5,
            "gemm_source_sha256": hashlib.sha256(src).hexdigest()}
    (root / "profiles" / "gemm_traffic.json").write_text(json.dumps(prof))
    monkeypatch.setattr(bench, "ROOT", str(root))
    got = bench.gemm_profile()
    assert got["traffic_bytes_per_launch"] == 1234567 and got["tensor_pipe_pct"] == 71.5
    (root / "nvfp4_bit_microscaled_b200" / "csrc" / "gemm.cu").write_bytes(src + b"// changed\n")
    assert bench.gemm_profile() is None


def test_committed_gemm_profile_is_well_formed():
    path = os.path.join(bench.ROOT, bench.GEMM_PROFILE)
    if not os.path.exists(path):
        return
    prof = json.load(open(path))
    assert prof["traffic_bytes_per_launch"] > 0 and 0 < prof["tensor_pipe_pct"] <= 100
    assert re.fullmatch(r"[0-9a-f]{64}", prof["gemm_source_sha256"])
    assert str(bench.WORKLOAD["T"]) in prof["workload"]


def test_both_arms_print_the_same_config():
    c1, c8 = bench.workload_config(1), bench.workload_config(8)
    assert c1["T"] == bench.WORKLOAD["T"] and c1["Cin"] == bench.WORKLOAD["Cin"]
    assert c1["Cout"] == bench.WORKLOAD["Cout"]
    assert c8["parallelism"].startswith("dp8") and c1["workload"] == c8["workload"]


def test_headline_is_the_largest_configuration():
    work = {k: w["T"] * w["Cin"] * w["Cout"] for k, w in bench.WORKLOADS.items()}
    assert bench.HEADLINE == max(work, key=work.get)


def test_fp4_roofline_uses_the_burst_bf16_figure():
    peaks = {"hbm_gbs": 6457.1, "bf16_tflops": 1698.2, "bf16_tflops_sustained": 1430.9}
    v, src = bench.fp4_peak(peaks, "measured")
    assert v == 4 * 1698.2 and "burst" in src
