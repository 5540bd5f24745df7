"""The benchmark's clock record, against a fake NVML: the sampler reads the SM
clock, its maximum and the clock-event (throttle) reasons during the timed
region only, reports the median clock and every reason seen, and never calls
anything that sets or resets a GPU setting."""
import sys
import time
import types

import pytest

import bench


class _FakeNvml(types.ModuleType):
    HW, HW_THERMAL, SW_THERMAL, SW_POWER = 0x8, 0x40, 0x20, 0x4

    def __init__(self, clocks, reasons):
        super().__init__("pynvml")
        self.calls = []
        self._clocks, self._reasons, self._i = clocks, reasons, 0
        self.NVML_CLOCK_SM = 1
        self.nvmlClocksEventReasonHwSlowdown = self.HW
        self.nvmlClocksEventReasonHwThermalSlowdown = self.HW_THERMAL
        self.nvmlClocksEventReasonSwThermalSlowdown = self.SW_THERMAL
        self.nvmlClocksEventReasonSwPowerCap = self.SW_POWER

    def nvmlInit(self):
        self.calls.append("nvmlInit")

    def nvmlDeviceGetHandleByPciBusId(self, pci):
        self.calls.append("nvmlDeviceGetHandleByPciBusId")
        return ("handle", pci)

    def nvmlDeviceGetHandleByIndex(self, i):
        self.calls.append("nvmlDeviceGetHandleByIndex")
        return ("handle", i)

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls.append("nvmlDeviceGetClockInfo")
        v = self._clocks[self._i % len(self._clocks)]
        self._i += 1
        return v

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        self.calls.append("nvmlDeviceGetMaxClockInfo")
        return 1965

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        self.calls.append("nvmlDeviceGetCurrentClocksEventReasons")
        return self._reasons

    def __getattr__(self, name):
        # any other NVML call (a setter, a reset) is recorded and refused
        if name.startswith("nvml"):
            def refused(*a, **k):
                self.calls.append(name)
                raise AssertionError(f"the clock sampler called {name}")
            return refused
        raise AttributeError(name)


@pytest.fixture
def fake_nvml(monkeypatch):
    def make(clocks, reasons):
        fake = _FakeNvml(clocks, reasons)
        monkeypatch.setitem(sys.modules, "pynvml", fake)
        return fake
    return make


def _sample(period=0.002, run_s=0.1):
    s = bench.ClockSampler(0, "00000000:1B:00.0", period_s=period)
    s.start()
    time.sleep(0.02)                  # samples before the region are not counted
    t0 = time.time()
    time.sleep(run_s)
    t1 = time.time()
    time.sleep(0.02)
    return s.stop(t0, t1)


def test_median_clock_and_power_cap_reason(fake_nvml):
    fake = fake_nvml([1965, 1950, 1965, 1940, 1965], _FakeNvml.SW_POWER)
    r = _sample()
    assert r["source"] == "nvml, 10 ms" and r["samples"] >= 5
    assert r["sm_mhz"] in (1940, 1950, 1965) and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]
    assert set(fake.calls) <= {"nvmlInit", "nvmlDeviceGetHandleByPciBusId",
                               "nvmlDeviceGetClockInfo", "nvmlDeviceGetMaxClockInfo",
                               "nvmlDeviceGetCurrentClocksEventReasons"}


def test_every_throttle_reason_is_reported(fake_nvml):
    fake_nvml([1200], _FakeNvml.HW | _FakeNvml.HW_THERMAL | _FakeNvml.SW_THERMAL)
    r = _sample()
    assert r["sm_mhz"] == 1200
    assert r["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_reason_when_none_is_active(fake_nvml):
    fake_nvml([1965], 0)
    r = _sample()
    assert r["reasons"] == [] and r["sm_mhz"] == 1965


def test_only_samples_inside_the_region_count(fake_nvml):
    fake_nvml([1965], 0)
    s = bench.ClockSampler(0, None, period_s=0.002)
    s.start()
    time.sleep(0.05)
    t = time.time()
    r = s.stop(t + 10.0, t + 20.0)      # a region in which nothing was sampled
    assert r["samples"] == 0 and r["sm_mhz"] is None and r["reasons"] == ["no samples"]
