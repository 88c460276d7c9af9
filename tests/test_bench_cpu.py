"""Host-side pieces of bench.py, without a GPU: the clock sampler against a fake NVML."""
import sys
import time
import types

import bench


def _fake_nvml(clocks, reasons):
    """A stand-in for pynvml that reports the given SM clocks and reason bit masks in turn
    and records that it was shut down; it exposes reads only."""
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    state = {"i": 0, "shutdown": False}

    def nvmlInit():
        pass

    def nvmlShutdown():
        state["shutdown"] = True

    def nvmlDeviceGetHandleByUUID(u):
        assert u.startswith("GPU-")
        return "h"

    def nvmlDeviceGetHandleByIndex(i):
        return "h"

    def nvmlDeviceGetMaxClockInfo(h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(h, kind):
        return clocks[min(state["i"], len(clocks) - 1)]

    def nvmlDeviceGetCurrentClocksEventReasons(h):
        r = reasons[min(state["i"], len(reasons) - 1)]
        state["i"] += 1
        return r

    for f in (nvmlInit, nvmlShutdown, nvmlDeviceGetHandleByUUID, nvmlDeviceGetHandleByIndex,
              nvmlDeviceGetMaxClockInfo, nvmlDeviceGetClockInfo,
              nvmlDeviceGetCurrentClocksEventReasons):
        setattr(m, f.__name__, f)
    return m, state


def test_clock_sampler_reads_nvml(monkeypatch):
    # 0x4: sw_power_cap, 0x40: hw_thermal_slowdown, 0x1 (idle) is not a reported reason
    fake, state = _fake_nvml([1965, 1800, 1700], [0x1, 0x4, 0x44])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(uuid="1234-abcd"))
    with bench.ClockSampler(0) as clk:
        deadline = time.time() + 5
        while len(clk.samples) < 5 and time.time() < deadline:
            time.sleep(0.01)
    s = clk.summary()
    assert s["source"] == "nvml" and s["samples"] >= 5
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] == 1700
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert state["shutdown"]


def test_clock_sampler_without_samples_says_so():
    s = bench.ClockSampler(0).summary()
    assert s["sm_mhz"] is None and s["reasons"] == ["clocks not sampled"]
