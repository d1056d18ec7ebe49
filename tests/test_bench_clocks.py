"""bench.py's clock sampler on the CPU against a fake NVML: samples are summarised over
the timed window only, and clock-event reasons are reported with their sample counts.
Nothing here reads or sets a real GPU."""
import sys
import time
import types

import bench


class _FakeNvml(types.ModuleType):
    """Reports 1965 MHz outside the window and 1500 MHz with the power cap inside it."""

    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    class NVMLError(Exception):
        pass

    def __init__(self):
        super().__init__("pynvml")
        self.loaded = False
        self.hot = False

    def nvmlInit(self):
        self.loaded = True

    def nvmlDeviceGetHandleByUUID(self, uuid):
        assert uuid == "GPU-fake"
        return object()

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        return 1500 if self.hot else 1965

    def nvmlDeviceGetPowerUsage(self, h):
        return 990_000 if self.hot else 200_000

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.nvmlClocksEventReasonSwPowerCap if self.hot else 0


def test_sampler_summarises_the_timed_window(monkeypatch):
    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler("GPU-fake", period_s=0.002)
    s.start()
    assert fake.loaded and s.samples, "start returns after the first sample"
    time.sleep(0.05)
    fake.hot = True
    time.sleep(0.01)
    s.begin()
    time.sleep(0.2)
    s.end()
    fake.hot = False
    time.sleep(0.05)
    clk = s.stop()
    assert clk["samples"] >= 20
    assert clk["sm_mhz"] == 1500 and clk["sm_max_mhz"] == 1965 and clk["power_w_max"] == 990
    assert clk["reasons"] == ["sw_power_cap"] and clk["reason_samples"]["sw_power_cap"] == clk["samples"]
    assert not bench.clocks_rejected(clk)  # the power cap is kept and noted


def test_rejection_rules():
    assert bench.clocks_rejected({"reasons": ["hw_thermal_slowdown"], "sm_mhz": 1900, "sm_max_mhz": 1965})
    assert bench.clocks_rejected({"reasons": [], "sm_mhz": 700, "sm_max_mhz": 1965})  # a leftover lock
    assert not bench.clocks_rejected({"reasons": ["sw_power_cap"], "sm_mhz": 1300, "sm_max_mhz": 1965})
