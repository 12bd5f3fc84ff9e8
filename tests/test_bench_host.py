"""Host logic of bench.py that needs no GPU: the clock sampler against a fake
NVML (the median SM clock and the clock-event reasons seen inside the timed
window, which decide whether a run is kept), the roofline denominators, the
algorithmic bytes and FLOPs of the kernel and step rooflines (weights and x
once, no padded or round-trip traffic), the source-hash gate on recorded DRAM
bytes, and the kernel count per forward.
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


PEAKS = {"hbm_gbs": 6537.0, "bf16_tflops": 1627.7, "bf16_tflops_sustained": 1372.1, "source": "measured"}


def _res(stage_ms, live, routes, touched, timed_s=0.05):
    return {"stage_ms": stage_ms, "live": live, "routes": routes, "touched": touched, "timed_s": timed_s,
            "ms_per_step": sum(stage_ms.values())}


def test_kernel_roofline_counts_weights_and_x_once(monkeypatch):
    """Decode shapes: the gate/up GEMM's algorithmic bytes are W1 of the touched
    experts plus x of the live tokens, once each (no route-row or h traffic)."""
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    w = bench.workloads.WORKLOADS["decode"]
    res = _res({"route": 0.008, "permute": 0.011, "gemm_gate_up": 0.165, "gemm_down": 0.087, "combine": 0.009},
               live=256, routes=2048, touched=128)
    r = bench.roofline(w, res, PEAKS)
    assert r["kernel"] == "gemm_gate_up" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["algorithmic_per_launch"] == 128 * 2 * 1024 * 2048 * 2 + 256 * 2048 * 2 == 1_074_790_400
    assert abs(r["achieved"] - 1_074_790_400 / 0.165e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6537.0) < 1e-12


def test_kernel_roofline_is_tensor_bound_at_prefill_and_picks_the_peak_by_duration(monkeypatch):
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    w = bench.workloads.WORKLOADS["prefill"]
    st = {"route": 0.024, "permute": 0.023, "gemm_gate_up": 0.95, "gemm_down": 0.55, "combine": 0.19}
    r = bench.roofline(w, _res(st, live=16384, routes=131072, touched=128), PEAKS)
    flops = 2.0 * 2 * 131072 * 2048 * 1024
    assert r["bound"] == "tensor" and r["algorithmic_per_launch"] == flops
    assert r["peak"] == 1627.7 and r["peak_kind"] == "burst bf16"
    assert abs(r["achieved"] - flops / 0.95e-3 / 1e12) < 1e-6
    # a timed region of more than a second is held to the sustained peak
    r2 = bench.roofline(w, _res(st, live=16384, routes=131072, touched=128, timed_s=2.0), PEAKS)
    assert r2["peak"] == 1372.1 and r2["peak_kind"] == "sustained bf16"
    # MXFP8 sits at the ridge: the FLOPs' time at twice the bf16 peak (the nominal fp8 / bf16
    # ratio) against the E4M3 weights' and scales' time, which grows with the touched experts
    wm = bench.workloads.WORKLOADS["mxfp8"]
    r3 = bench.roofline(wm, _res(st, live=4096, routes=32768, touched=120), PEAKS)
    assert r3["bound"] == "tensor" and abs(r3["peak"] - 2 * 1627.7) < 1e-9
    r4 = bench.roofline(wm, _res(st, live=4096, routes=32768, touched=128), PEAKS)
    assert r4["bound"] == "hbm"
    assert r4["algorithmic_per_launch"] == 128 * 2 * 1024 * 2048 * (1 + 1 / 32) + 4096 * 2048 * (1 + 1 / 32)


def test_step_roofline_of_the_decode_step(monkeypatch):
    """Every expert's three projections once, plus per live token x in, logits
    in and the fp32 output out; the roofline time is the larger of the bytes'
    and the FLOPs' times."""
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    w = bench.workloads.WORKLOADS["decode"]
    res = _res({"gemm_gate_up": 0.165, "gemm_down": 0.0866}, live=256, routes=2048, touched=128)
    res["ms_per_step"] = 0.2543
    s = bench.step_roofline(w, res, PEAKS)
    bytes_ = 128 * 3 * 2048 * 1024 * 2 + 256 * (2048 * 2 + 128 * 4 + 2048 * 4)
    assert s["bytes"] == bytes_ == 1_613_889_536 and s["bound"] == "hbm"
    assert abs(s["roofline_ms"] - bytes_ / 6537e9 * 1e3) < 1e-12
    assert abs(s["frac_burst"] - s["roofline_ms"] / 0.2543) < 1e-12
    assert s["flops"] == 2.0 * 3 * 2048 * 2048 * 1024


def test_recorded_traffic_only_for_unchanged_sources(monkeypatch):
    """The committed DRAM bytes are reported only while the kernel's sources
    hash to the value recorded beside them."""
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    import json

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)["gemm_gate_up@decode"]
    monkeypatch.setattr(bench, "source_hash", lambda stage, precision: rec["source_sha"])
    assert bench.recorded_traffic("gemm_gate_up", "decode", "bf16") == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "source_hash", lambda stage, precision: "0" * 16)
    assert bench.recorded_traffic("gemm_gate_up", "decode", "bf16") is None
    assert bench.recorded_traffic("gemm_gate_up", "no-such-workload", "bf16") is None


def test_kernel_launch_counts_per_forward(monkeypatch):
    """route, permute, gate/up, down, combine; MXFP8 adds the quantising gather,
    NVFP4 the gather and the h pass."""
    bench = _bench(monkeypatch, _fake_nvml([1965], [0]))
    assert bench.kernels_per_forward("bf16", 65536) == 5
    assert bench.kernels_per_forward("mxfp8", 4096) == 6
    assert bench.kernels_per_forward("nvfp4", 4096) == 7
