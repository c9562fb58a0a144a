"""Host tests of the bench's clock sampling: the NVML poller that reads the SM
clock and the active clocks-event reasons while the timed steps run (a timed
region of a millisecond sees no 200 ms nvidia-smi sample). A fake NVML module
stands in for the driver's; nothing here needs or touches a GPU."""
import os
import sys
import time

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, uuids, sm=1965, max_sm=1965, bits=0, fail_init=False):
        self.uuids, self.sm, self.max_sm, self.bits = uuids, sm, max_sm, bits
        self.fail_init = fail_init
        self.queried = set()
        self.shutdowns = 0

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no NVML")

    def nvmlShutdown(self):
        self.shutdowns += 1

    def nvmlDeviceGetCount(self):
        return len(self.uuids)

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetUUID(self, h):
        return "GPU-" + self.uuids[h]

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        self.queried.add(h)
        return self.sm

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return self.max_sm

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.bits


def sample(nv, uuid=None, index=0, seconds=0.02):
    with bench.ClockSampler(index, uuid, nvml=nv) as clk:
        time.sleep(seconds)
    return clk.summary()


def test_nvml_samples_the_device_with_the_cuda_uuid():
    nv = FakeNvml(["aaaa", "bbbb", "cccc"], sm=1965, bits=0x1 | 0x4)  # idle + sw power cap
    s = sample(nv, uuid="cccc", index=0)
    assert nv.queried == {2}                  # matched by UUID, not by index 0
    assert s["nvml_samples"] >= 3 and s["samples"] >= s["nvml_samples"]
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["sm_mhz_min"] == 1965
    assert s["reasons"] == ["sw_power_cap"]   # idle is not a slowdown
    assert nv.shutdowns == 1


def test_nvml_reason_bits_map_to_the_reported_names():
    nv = FakeNvml(["aaaa"], bits=0x8 | 0x20 | 0x40 | 0x80)
    s = sample(nv, uuid="GPU-AAAA")
    assert s["reasons"] == ["hw_power_brake_slowdown", "hw_slowdown", "hw_thermal_slowdown",
                            "sw_thermal_slowdown"]


def test_nvml_falls_back_to_the_index_without_a_uuid():
    nv = FakeNvml(["aaaa", "bbbb"], sm=1500, max_sm=1965)
    s = sample(nv, uuid=None, index=1)
    assert nv.queried == {1}
    assert s["sm_mhz"] == 1500 and s["sm_max_mhz"] == 1965


def test_no_nvml_leaves_no_samples_and_no_error():
    s = sample(FakeNvml(["aaaa"], fail_init=True))
    assert s["nvml_samples"] == 0
    if s["smi_samples"] == 0:  # no nvidia-smi on this host either
        assert s["sm_mhz"] is None and s["samples"] == 0
