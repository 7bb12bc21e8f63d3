"""bench.py's clock sampler against a stand-in NVML (no GPU needed): it reads
the SM clock and the clock-event reasons on a thread while the region runs,
reports the median clock and every throttle reason seen, and degrades to
"unsampled" when NVML is not usable.  It only reads; nothing is set."""
import time

import bench


class FakeNVML:
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons, fail_init=False):
        self.clocks, self.reasons, self.fail_init = clocks, reasons, fail_init
        self.i = 0
        self.calls = []

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no NVML")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByUUID(self, uuid):
        self.calls.append(("uuid", uuid))
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self.clocks[min(self.i, len(self.clocks) - 1)]
        self.i += 1
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons[min(self.i - 1, len(self.reasons) - 1)]


def test_median_clock_and_reasons_seen_during_the_region():
    nv = FakeNVML([1965, 1965, 1800, 1965, 1965], [0, 0x4, 0x4, 0, 0])
    with bench.ClockSampler("GPU-abc", nvml=nv, period_s=0.001) as clk:
        time.sleep(0.05)
    s = clk.summary()
    assert s["samples"] >= 3
    assert s["sm_max_mhz"] == 1965
    assert s["sm_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert ("uuid", "GPU-abc") in nv.calls and "shutdown" in nv.calls


def test_thermal_and_hw_slowdown_are_reported():
    nv = FakeNVML([1400], [0x8 | 0x40 | 0x20])
    with bench.ClockSampler("GPU-x", nvml=nv, period_s=0.001) as clk:
        time.sleep(0.02)
    assert clk.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown",
                                        "sw_thermal_slowdown"]


def test_unusable_nvml_gives_unsampled():
    with bench.ClockSampler("GPU-x", nvml=FakeNVML([1], [0], fail_init=True)) as clk:
        pass
    assert clk.summary()["reasons"] == ["unsampled"]
