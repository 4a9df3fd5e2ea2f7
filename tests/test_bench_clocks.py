"""bench.py's clock sampler against a fake NVML (no GPU): it reads SM clocks and throttle reasons
only (it sets nothing), reports their median and the union of reasons by name, leaves out
gpu_idle, and reports no clocks rather than guessing when NVML is missing."""
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_nvml(clocks, reasons, calls):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    state = {"i": 0}

    def record(name):
        calls.append(name)

    nv.nvmlInit = lambda: record("init")
    nv.nvmlDeviceGetHandleByIndex = lambda i: (record("handle"), ("dev", i))[1]
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        i = state["i"]
        state["i"] += 1
        return clocks[i % len(clocks)]

    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[state["i"] % len(reasons)]

    def other(name):  # any other NVML call (a setter, a reset) is recorded and refused
        record("other:" + name)
        raise AttributeError(name)

    nv.__getattr__ = other
    return nv


def test_median_clock_and_reason_names(monkeypatch):
    calls = []
    fake = _fake_nvml([1965, 1950, 1965, 1800, 1965], [0x1, 0x4, 0x0, 0x8], calls)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0, period_s=0.001) as clk:
        time.sleep(0.05)
    rep = clk.report()
    assert rep["sm_max_mhz"] == 1965 and rep["samples"] > 0
    assert 1800 <= rep["sm_mhz"] <= 1965
    assert "sw_power_cap" in rep["reasons"] and "hw_slowdown" in rep["reasons"]
    assert "gpu_idle" not in rep["reasons"]
    # only the read calls above: nothing else of NVML was touched
    assert not [c for c in calls if c.startswith("other:")], calls


def test_no_nvml_reports_no_clocks(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    with bench.ClockSampler(0) as clk:
        pass
    rep = clk.report()
    assert rep == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
