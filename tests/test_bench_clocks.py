"""CPU checks of bench.py's clock record and launch count.  The clock sampler
reads NVML (never sets anything); here a fake NVML stands in for the driver,
so the checks need no GPU: only samples inside the timed regions count, the
clock-event reason bits map to their names, the older throttle-reasons call
is used where the event-reasons one is missing, and a failing NVML falls back
to nvidia-smi (or reports that no clock source exists)."""
import time

import pytest

import bench
import synth


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, event_call=True, fail_init=False):
        self.sm, self.bits = 1965, 0
        self.event_call, self.fail_init = event_call, fail_init
        self.calls = []

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no NVML")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByUUID(self, u):
        if u != "GPU-1234":
            raise RuntimeError("unknown uuid")
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        return "h"

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        if not self.event_call:
            raise RuntimeError("function not found")
        self.calls.append("event")
        return self.bits

    def nvmlDeviceGetCurrentClocksThrottleReasons(self, h):
        self.calls.append("throttle")
        return self.bits

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        assert which == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        assert which == self.NVML_CLOCK_SM
        return self.sm


# State changes sit 50 ms away from the region's edges: a sample's time stamp
# and its reading are two steps of the polling thread, which the interpreter
# may separate by a thread switch (5 ms by default).
GAP = 0.05


def _run(sampler, fake):
    sampler.start()
    fake.sm, fake.bits = 1965, 0x8            # hw_slowdown outside the timed regions: not counted
    time.sleep(GAP)
    fake.sm, fake.bits = 1900, 0x4            # sw_power_cap inside
    time.sleep(GAP)
    sampler.begin()
    time.sleep(2 * GAP)
    sampler.end()
    time.sleep(GAP)
    fake.sm, fake.bits = 1500, 0x40           # thermal slowdown after: not counted
    time.sleep(GAP)
    return sampler.stop()


def test_nvml_samples_only_inside_timed_regions(monkeypatch):
    fake = FakeNvml()
    monkeypatch.setattr(bench, "_load_nvml", lambda: fake)
    c = _run(bench.ClockSampler(0, "1234"), fake)
    assert c["source"].startswith("NVML")
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples"] >= 3
    assert "event" in fake.calls and "throttle" not in fake.calls and fake.calls[-1] == "shutdown"


def test_nvml_throttle_call_when_event_call_is_missing(monkeypatch):
    fake = FakeNvml(event_call=False)
    monkeypatch.setattr(bench, "_load_nvml", lambda: fake)
    c = _run(bench.ClockSampler(0, "unknown-uuid"), fake)   # falls back to the index handle
    assert c["reasons"] == ["sw_power_cap"] and c["sm_mhz"] == 1900
    assert "throttle" in fake.calls


def test_reason_bits_map_to_names(monkeypatch):
    fake = FakeNvml()
    monkeypatch.setattr(bench, "_load_nvml", lambda: fake)
    s = bench.ClockSampler(0)
    s.start()
    fake.bits = 0x8 | 0x20 | 0x40 | 0x4 | 0x1   # 0x1 (idle) is not reported
    time.sleep(GAP)
    s.begin()
    time.sleep(2 * GAP)
    s.end()
    c = s.stop()
    assert c["reasons"] == sorted(["hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown", "sw_power_cap"])


def test_failing_nvml_falls_back(monkeypatch):
    fake = FakeNvml(fail_init=True)
    monkeypatch.setattr(bench, "_load_nvml", lambda: fake)
    s = bench.ClockSampler(0)
    s.start()
    assert s.nv is None
    s.begin()
    s.end()
    c = s.stop()
    # nvidia-smi takes over; on a machine without it (or without a GPU) no sample is taken
    assert c["samples"] == 0 or c["source"].startswith("nvidia-smi")


@pytest.mark.parametrize("path,want", [(0, 4), (1, 7), (2, 6)], ids=["gemv", "warp_mma", "tcgen05"])
def test_launches_per_step(path, want):
    """Router + shared down + the routed experts' kernels of each path (the
    path itself comes from moe_layer_expert_path)."""
    for cfg_id in (1, 2, 3):
        b = synth.CONFIGS[cfg_id].batch
        extra = (1 if path == 2 and b > 1 else 0) + (1 if path == 2 and b > 2 else 0)  # routing finish, combine
        want_c = want + extra
        assert bench.launches_per_step(synth.CONFIGS[cfg_id], path) == want_c
        assert bench.launches_per_step(synth.CONFIGS[cfg_id].with_(shared_inter=0), path) == want_c - 1
        assert bench.launches_per_step(synth.CONFIGS[cfg_id].with_(shared_format="mxfp4"), path) == want_c + 1
