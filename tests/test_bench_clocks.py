"""bench.py's clock sampler on a fake NVML: several samples in a short region, reasons decoded from
the clock-event bit mask, and nothing but reads issued."""
import sys
import time
import types

import bench


def fake_nvml(clocks, reasons):
    calls = []
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    state = {"i": 0}

    def rec(name):
        def f(*a):
            calls.append(name)
            if name == "clock":
                state["i"] += 1
                return clocks[min(state["i"] - 1, len(clocks) - 1)]
            if name == "reasons":
                return reasons[min(state["i"] - 1, len(reasons) - 1)]
            if name == "max":
                return 1965
            return object()
        return f

    nv.nvmlInit = rec("init")
    nv.nvmlDeviceGetHandleByIndex = rec("handle")
    nv.nvmlDeviceGetHandleByPciBusId = rec("handle")
    nv.nvmlDeviceGetMaxClockInfo = rec("max")
    nv.nvmlDeviceGetClockInfo = rec("clock")
    nv.nvmlDeviceGetCurrentClocksEventReasons = rec("reasons")
    return nv, calls


def test_sampler_reports_median_and_reasons(monkeypatch):
    nv, calls = fake_nvml([1965, 1965, 1900, 1965] + [1965] * 100, [0x0, 0x4, 0x0, 0x1] + [0x0] * 100)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    with bench.ClockSampler(0) as s:
        time.sleep(0.05)
    out = s.summary()
    assert out["samples"] >= 4
    assert out["sm_mhz"] == 1965 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]          # 0x1 (idle) is not a slowdown reason
    assert set(calls) <= {"init", "handle", "max", "clock", "reasons"}


def test_sampler_flags_thermal_and_hw_slowdown(monkeypatch):
    nv, _ = fake_nvml([1200] * 50, [0x8 | 0x40 | 0x20] * 50)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    with bench.ClockSampler(0) as s:
        time.sleep(0.03)
    assert s.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
