"""The benchmark's clock sampler on CPU, against a fake NVML (reads only; nothing is set)."""
import os
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_nvml(clocks, reasons, fail_init=False):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    state = {"i": 0, "shutdown": 0}

    def init():
        if fail_init:
            raise RuntimeError("no driver")
    m.nvmlInit = init
    m.nvmlShutdown = lambda: state.__setitem__("shutdown", state["shutdown"] + 1)
    m.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[state["i"] % len(clocks)]
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[state["i"] % len(reasons)]
    return m, state


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_nvml_samples_and_reasons(monkeypatch):
    fake, state = _fake_nvml([1965, 1900, 1965], [0, 0x4, 0])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench = _bench()
    with bench.ClockSampler(0) as clk:
        time.sleep(0.15)
    s = clk.summary()
    assert s["source"] == "nvml"
    assert s["samples"] >= 5
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] in (1900.0, 1965.0)
    assert s["reasons"] == ["sw_power_cap"]
    assert state["shutdown"] == 1


def test_hw_reasons_are_reported(monkeypatch):
    fake, _ = _fake_nvml([1200], [0x8 | 0x40])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench = _bench()
    with bench.ClockSampler(0) as clk:
        time.sleep(0.05)
    assert clk.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_without_nvml_or_nvidia_smi_the_summary_is_empty(monkeypatch):
    fake, _ = _fake_nvml([1965], [0], fail_init=True)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setenv("PATH", "/nonexistent")
    bench = _bench()
    with bench.ClockSampler(0) as clk:
        pass
    s = clk.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None and s["source"] is None
