"""The bench's clock record (CPU, against a fake NVML): the SM clock, power and
clock-event reasons come from samples taken inside the timed region only, the
GPU is found by UUID (by index when the UUID is unknown), and a missing NVML
leaves the nvidia-smi path alone."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, uuid="GPU-0000", fail_init=False):
        self.uuid, self.fail_init = uuid, fail_init
        self.clock, self.reasons, self.by_index = 1500, 0, []

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no NVML")

    def nvmlDeviceGetHandleByUUID(self, u):
        if u != self.uuid:
            raise RuntimeError("unknown uuid")
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        self.by_index.append(i)
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.clock

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons

    def nvmlDeviceGetPowerUsage(self, h):
        return 950_000   # mW


def test_only_region_samples_count():
    nv = FakeNvml()
    s = bench.ClockSampler(0, "GPU-0000", nvml=nv)
    s.start()
    nv.clock, nv.reasons = 1100, 0x8          # outside the region: ignored
    time.sleep(0.03)
    nv.clock, nv.reasons = 1900, 0x4          # inside: sw_power_cap
    s.begin()
    time.sleep(0.08)
    s.end()
    nv.clock, nv.reasons = 1000, 0x40
    time.sleep(0.03)
    r = s.stop()
    assert r["region_samples"] >= 10
    assert r["sm_mhz"] == 1900 and r["sm_max_mhz"] == 1965
    assert "sw_power_cap" in r["reasons"]
    assert "hw_slowdown" not in r["reasons"] and "hw_thermal_slowdown" not in r["reasons"]
    assert r["power_w_max"] == 950.0


def test_unknown_uuid_falls_back_to_the_index():
    nv = FakeNvml(uuid="GPU-1111")
    s = bench.ClockSampler(3, "GPU-2222", nvml=nv)
    s.start()
    s.begin()
    time.sleep(0.02)
    s.end()
    r = s.stop()
    assert nv.by_index == [3] and s.uuid is None
    assert r["region_samples"] >= 1


def test_without_nvml_the_record_still_forms():
    s = bench.ClockSampler(0, None, nvml=FakeNvml(fail_init=True))
    s.start()
    s.begin()
    s.end()
    r = s.stop()
    assert set(r) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    assert s.handle is None and r.get("region_samples", 0) == 0
