"""The bench's SM clock record, on CPU against a fake NVML module.

The sampler must keep reading clocks until the timed steps have drained from the GPU (polled
through a CUDA event), map the throttle-reason bits to names, leave `gpu_idle` out, and report
the absence of NVML instead of guessing a clock.
"""
import sys
import types

import pytest


class _FakeNvml(types.ModuleType):
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, mask, fail=False):
        super().__init__("pynvml")
        self._clocks, self._mask, self._fail, self.reads = list(clocks), mask, fail, 0

    def nvmlInit(self):
        if self._fail:
            raise RuntimeError("NVML Shared Library Not Found")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("handle", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.reads += 1
        return self._clocks[(self.reads - 1) % len(self._clocks)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self._mask


class _Event:
    """Completes after `n` polls, like a CUDA event behind queued work."""

    def __init__(self, n):
        self.n = n

    def query(self):
        self.n -= 1
        return self.n < 0


@pytest.fixture
def bench_with(monkeypatch):
    def make(fake):
        monkeypatch.setitem(sys.modules, "pynvml", fake)
        import bench
        return bench
    return make


def test_sampler_polls_until_the_event_completes(bench_with):
    fake = _FakeNvml([1965, 1800, 1900], mask=0x1 | 0x4)   # gpu_idle + sw_power_cap
    bench = bench_with(fake)
    s = bench.ClockSampler(0, period_s=0.0)
    with s:
        s.wait(_Event(12))
    out = s.summary()
    assert out["samples"] >= 12            # the waiting thread alone reads 12 times
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert out["sm_mhz_range"] == [1800, 1965]
    assert out["sm_mhz"] in (1800, 1900, 1965)


def test_sampler_maps_every_reason_bit(bench_with):
    fake = _FakeNvml([1500], mask=0x8 | 0x20 | 0x40)
    bench = bench_with(fake)
    s = bench.ClockSampler(0, period_s=0.0)
    with s:
        s.wait(_Event(3))
    assert s.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_sampler_without_nvml_reports_no_clock(bench_with):
    bench = bench_with(_FakeNvml([1965], mask=0, fail=True))
    s = bench.ClockSampler(0, period_s=0.0)
    with s:
        s.wait(_Event(2))
    out = s.summary()
    assert out["sm_mhz"] is None and out["sm_max_mhz"] is None
    assert "NVML" in out["note"]
