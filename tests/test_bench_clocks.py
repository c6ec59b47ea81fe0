"""bench.py's clock record, on a fake NVML (CPU only): samples are taken while
the timed region runs (from begin() until its last event completes), and the
record names the clock-event reasons that were active."""
import sys
import time
import types

import pytest


@pytest.fixture
def fake_nvml(monkeypatch):
    calls = {"clock": 0}
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlInit = lambda: None
    nv.nvmlShutdown = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda uuid: "handle"
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        calls["clock"] += 1
        return 1800 if calls["clock"] % 2 else 1965

    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetPowerUsage = lambda h: 612000          # mW
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 | 0x40   # power cap, hw thermal
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    return calls


class _Event:
    """Stands in for a CUDA event that completes after `seconds`."""

    def __init__(self, seconds):
        self.t = time.monotonic() + seconds

    def query(self):
        return time.monotonic() >= self.t


def test_samples_cover_the_region_and_name_the_reasons(fake_nvml):
    import bench
    c = bench.ClockSampler("GPU-test")
    c.start()
    time.sleep(0.02)                  # before begin(): nothing is recorded
    assert c.samples == []
    c.begin()
    c.wait(_Event(0.03))
    rec = c.stop()
    assert rec["samples"] >= 5
    assert rec["sm_max_mhz"] == 1965
    assert rec["sm_min_mhz"] == 1800
    assert rec["power_w_max"] == pytest.approx(612.0)
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    n = rec["samples"]
    time.sleep(0.02)                  # after the region: the thread has stopped
    assert len(c.samples) == n


def test_region_shorter_than_the_thread_period_still_sampled(fake_nvml):
    import bench
    c = bench.ClockSampler("GPU-test")
    c.start()
    c.begin()
    c.wait(_Event(0.002))
    assert c.stop()["samples"] >= 1
