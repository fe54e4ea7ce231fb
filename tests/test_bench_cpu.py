"""bench.py's host logic on the CPU: which bf16 peak a timed region is held to, the tensor
peak at a sampled clock, and the clock sampler's NVML path against a fake NVML (reads only)."""
from __future__ import annotations

import sys
import time
import types

import bench


def test_peak_choice_follows_the_timed_region():
    peaks = {"bf16_tflops": 1647.6, "bf16_tflops_sustained": 1375.3, "hbm_gbs": 6542.4}
    assert bench.pick_peak(peaks, 0.8) == (1647.6, "burst")
    assert bench.pick_peak(peaks, 3.0) == (1647.6, "burst")
    assert bench.pick_peak(peaks, 12.0) == (1375.3, "sustained")


def test_tensor_peak_at_clock():
    # 148 SMs x 8192 flop/clk at 1965 MHz
    assert abs(bench.tensor_peak_at(1965.0, 148) - 148 * 8192 * 1.965e9 / 1e12) < 1e-9
    assert abs(bench.tensor_peak_at(1000.0, 148) - 1212.416) < 1e-6


def test_clock_sampler_nvml_path(monkeypatch):
    calls = {"n": 0}

    def clock(h, which):
        calls["n"] += 1
        return 1300 + (calls["n"] % 3) * 100          # 1300 / 1400 / 1500 MHz

    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda u: "h",
        nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, w: 1965,
        nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetPowerUsage=lambda h: 950_000,   # milliwatts
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0x4 | 0x1,   # power cap, idle
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler("GPU-0000", period_s=0.002)
    s.start()
    time.sleep(0.1)
    c = s.stop()
    assert c["source"].startswith("nvml") and c["samples"] >= 5
    assert c["sm_max_mhz"] == 1965.0 and 1300 <= c["sm_mhz"] <= 1500
    assert c["reasons"] == ["sw_power_cap"]            # only the four named reasons
    assert abs(c["power_w_median"] - 950.0) < 1e-9
