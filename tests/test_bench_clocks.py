"""The benchmark's clock record on CPU, against a fake NVML: samples come
from the timed window only, reason bits decode to the names the benchmark
reports, and any NVML failure falls back to the nvidia-smi record."""

import time

import bench


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, masks, fail_init=False, fail_uuid=False):
        self.clocks, self.masks = clocks, masks
        self.fail_init, self.fail_uuid = fail_init, fail_uuid
        self.k = 0
        self.by = None
        self.shutdown = False

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no NVML")

    def nvmlDeviceGetHandleByUUID(self, uuid):
        if self.fail_uuid:
            raise RuntimeError("unknown uuid")
        self.by = ("uuid", uuid)
        return "h"

    def nvmlDeviceGetHandleByIndex(self, index):
        self.by = ("index", index)
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self.clocks[min(self.k, len(self.clocks) - 1)]
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        v = self.masks[min(self.k, len(self.masks) - 1)]
        self.k += 1
        return v

    def nvmlShutdown(self):
        self.shutdown = True


def test_window_and_reasons():
    nv = FakeNvml([1965, 1800, 1700], [0x0, 0x4, 0x4 | 0x8])
    s = bench.ClockSampler(0, uuid="GPU-x", nvml=nv)
    s.start()
    s.window_begin()
    time.sleep(0.15)
    s.window_end()
    rec = s.stop()
    assert nv.by == ("uuid", "GPU-x") and nv.shutdown
    assert rec["source"].startswith("nvml") and rec["samples"] >= 3
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert 1700.0 <= rec["sm_mhz"] <= 1965.0


def test_samples_outside_the_window_are_left_out():
    r = bench.NvmlClockReader(0, nvml=FakeNvml([1965], [0]))
    r.samples = [(1.0, 900.0, 0x20), (2.0, 1900.0, 0x0), (3.0, 1950.0, 0x4), (4.0, 500.0, 0x40)]
    r.max_mhz = 1965.0
    rec = r.summary(1.5, 3.5)
    assert rec["samples"] == 2 and rec["sm_mhz"] == 1925.0 and rec["reasons"] == ["sw_power_cap"]
    assert r.summary(5.0, 6.0) is None
    assert r.summary(None, None) is None


def test_uuid_lookup_falls_back_to_the_index():
    nv = FakeNvml([1965], [0], fail_uuid=True)
    r = bench.NvmlClockReader(3, uuid="GPU-y", nvml=nv)
    assert r.start()
    r.stop()
    assert nv.by == ("index", 3)


def test_nvml_failure_falls_back_to_nvidia_smi_record():
    s = bench.ClockSampler(0, nvml=FakeNvml([1965], [0], fail_init=True))
    s.start()
    s.window_begin()
    s.window_end()
    rec = s.stop()
    assert not rec.get("source", "").startswith("nvml")
    assert "sm_mhz" in rec and "reasons" in rec
