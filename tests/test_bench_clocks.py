"""bench.py's clock record: the NVML sampler (read-only calls only) against a fake NVML
module, including a timed region shorter than one polling interval.  CPU only."""

import importlib.util
import os
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def fake_nvml(clocks, reasons):
    """A stand-in for the NVML binding that serves the given clock and reason sequences and
    records every call; it has no setter, so any attempt to change a setting fails."""
    calls = []
    it = {"i": 0}

    def step():
        i = min(it["i"], len(clocks) - 1)
        it["i"] += 1
        return i

    m = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlClocksEventReasonSwPowerCap=0x4, nvmlClocksEventReasonHwSlowdown=0x8,
        nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonHwThermalSlowdown=0x40,
        calls=calls)
    state = {"last": 0}
    m.nvmlInit = lambda: calls.append("init")
    m.nvmlShutdown = lambda: calls.append("shutdown")

    def handle(u):
        calls.append(("handle", u))
        assert u.startswith("GPU-")
        return "h"

    def clock(h, kind):
        assert h == "h" and kind == 1
        state["last"] = step()
        return clocks[state["last"]]

    m.nvmlDeviceGetHandleByUUID = handle
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[state["last"]]
    return m


def test_nvml_sampler_median_and_reasons():
    bench = load_bench()
    clocks = [1965, 1500, 1480, 1510, 1490, 1500, 1495]
    reasons = [0, 0x4, 0x4, 0x4 | 0x8, 0x4, 0x4, 0x4]
    s = bench.NvmlClockSampler("abcd-1234", fake_nvml(clocks, reasons), period_s=0.001)
    s.start()
    time.sleep(0.05)
    rec = s.stop()
    assert rec["source"] == "nvml" and rec["samples"] >= 2
    assert rec["sm_max_mhz"] == 1965
    assert 1480 <= rec["sm_mhz"] <= 1510          # the pre-region sample is not counted
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert ("handle", "GPU-abcd-1234") in s.nvml.calls
    assert s.nvml.calls[-1] == "shutdown"


def test_nvml_sampler_short_region_has_a_sample():
    bench = load_bench()
    s = bench.NvmlClockSampler("GPU-x", fake_nvml([1965, 1965], [0, 0]), period_s=10.0)
    s.start()
    rec = s.stop()            # shorter than one polling period
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1965.0 and rec["reasons"] == []


def test_nvidia_smi_sampler_without_the_tool():
    bench = load_bench()
    s = bench.ClockSampler(0)
    s.proc = None
    rec = s.stop()
    assert rec["sm_mhz"] is None and rec["reasons"] == ["nvidia-smi unavailable"]


def test_peaks_fill_missing_keys_from_the_fallback(tmp_path):
    bench = load_bench()
    p = tmp_path / "peaks.json"
    p.write_text('{"hbm_gbs": 6400.0, "bf16_tflops": "n/a", "sm_max_mhz": 1965}')
    peaks, kinds = bench.load_peaks(str(p))
    assert peaks["hbm_gbs"] == 6400.0 and kinds["hbm_gbs"] == "measured"
    assert peaks["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"] and kinds["bf16_tflops"] == "fallback"
    assert kinds["bf16_tflops_sustained"] == "fallback"
    peaks, kinds = bench.load_peaks(str(tmp_path / "absent.json"))
    assert peaks == bench.FALLBACK_PEAKS and set(kinds.values()) == {"fallback"}
    p.write_text("{not json")
    assert bench.load_peaks(str(p))[0] == bench.FALLBACK_PEAKS
