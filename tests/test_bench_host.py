"""Host logic of bench.py that needs no GPU: the clock sampler against a fake
NVML (the median SM clock and the clock-event reasons seen inside the timed
window, which decide whether a run is kept), and the roofline denominators.
"""
from __future__ import annotations

import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_nvml(clocks, reasons):
    """A pynvml stand-in whose SM clock and reasons follow the given lists."""
    state = {"i": 0}
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: "h"
    m.nvmlDeviceGetHandleByIndex = lambda i: "h"
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        i = min(state["i"], len(clocks) - 1)
        return clocks[i]

    def why(h):
        i = min(state["i"], len(reasons) - 1)
        state["i"] += 1
        return reasons[i]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = why
    return m


def _bench(monkeypatch, nvml):
    monkeypatch.setitem(sys.modules, "pynvml", nvml)
    sys.path.insert(0, ROOT)
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    import bench

    return bench


def test_clock_sampler_reports_median_and_reasons_inside_the_window(monkeypatch):
    bench = _bench(monkeypatch, _fake_nvml([1965, 1500, 1965, 1800] * 50, [0, 0x4, 0, 0x40] * 50))
    s = bench.ClockSampler(0)
    assert s.ok
    s.start()
    t0 = time.perf_counter()
    time.sleep(0.08)
    t1 = time.perf_counter()
    s.stop()
    s.window = (t0, t1)
    out = s.summary()
    assert out["sm_max_mhz"] == 1965
    assert out["samples"] >= 3
    assert 1500 <= out["sm_mhz"] <= 1965
    assert set(out["reasons"]) == {"sw_power_cap", "hw_thermal_slowdown"}


def test_clock_sampler_without_reasons_reports_none(monkeypatch):
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    s = bench.ClockSampler(0)
    s.start()
    t0 = time.perf_counter()
    time.sleep(0.05)
    t1 = time.perf_counter()
    s.stop()
    s.window = (t0, t1)
    out = s.summary()
    assert out["reasons"] == [] and out["sm_mhz"] == 1965


def test_clock_sampler_short_window_takes_the_nearest_samples(monkeypatch):
    bench = _bench(monkeypatch, _fake_nvml([1700], [0x8]))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.05)
    s.stop()
    mid = s.samples[len(s.samples) // 2][0]
    s.window = (mid + 1e-7, mid + 2e-7)  # between two samples
    out = s.summary()
    assert out["samples"] == 2 and out["reasons"] == ["hw_slowdown"] and out["sm_mhz"] == 1700


def test_measured_peaks_come_from_the_measured_file_when_present(monkeypatch):
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    p = bench.measured_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert p["source"] == "measured" and p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    else:
        assert p == {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                     "source": "fallback"}
