"""bench.py's clock sampler against a fake NVML, on the CPU.

The sampler only reads: the SM clock, the maximum SM clock and the mask of active
clock-event reasons, which it decodes into the names the bench line reports.
"""
import sys
import time
import types

import bench


def _fake_nvml(mask_seq):
    m = types.SimpleNamespace()
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    state = {"i": 0}
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: ("pci", bus)
    m.nvmlDeviceGetHandleByIndex = lambda i: ("index", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        return 1900 + (state["i"] % 3) * 30

    def reasons(h):
        state["i"] += 1
        return mask_seq[min(state["i"] - 1, len(mask_seq) - 1)]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = reasons
    return m, state


def test_nvml_samples_are_decoded_into_reason_names(monkeypatch):
    fake, _ = _fake_nvml([0x0, 0x4, 0x4 | 0x40, 0x0])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.ClockSampler(0)
    t0 = time.time()
    deadline = t0 + 5.0
    while len(c.samples) < 6 and time.time() < deadline:
        time.sleep(0.005)
    t1 = time.time()
    c.stop()
    s = c.summary(t0 - 1.0, t1 + 1.0)
    assert s["source"].startswith("nvml")
    assert s["samples"] >= 4 and s["window"] == "timed region"
    assert s["sm_max_mhz"] == 1965.0 and 1900.0 <= s["sm_mhz"] <= 1960.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_summary_keeps_only_samples_inside_the_timed_region():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.source = "test"
    c.samples = [(1.0, 1965.0, 1965.0, set()), (2.0, 1900.0, 1965.0, {"sw_power_cap"}),
                 (3.0, 1950.0, 1965.0, set()), (9.0, 100.0, 1965.0, {"hw_slowdown"})]
    s = c.summary(0.5, 3.5)
    assert s["samples"] == 3 and s["sm_mhz"] == 1950.0 and s["reasons"] == ["sw_power_cap"]
    s = c.summary(4.0, 5.0)  # nothing inside: the whole run stands in, and says so
    assert s["samples"] == 0 and s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert s["window"].startswith("whole run")
