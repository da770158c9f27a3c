"""bench.py's clock sampler against a fake NVML (CPU): the reasons it
reports, the median over samples under load, and the fallback when NVML
cannot start."""
import time

import bench


class FakeNvml:
    """The read-only pynvml calls the sampler makes; replays (MHz, reason
    bits) samples and then repeats the last one."""
    NVML_CLOCK_SM = 1

    def __init__(self, samples, max_mhz=1965):
        self.samples = list(samples)
        self.max_mhz = max_mhz
        self.i = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, uuid):
        assert uuid.startswith("GPU-")
        return object()

    def nvmlDeviceGetHandleByIndex(self, i):
        return object()

    def nvmlDeviceGetMaxClockInfo(self, h, clock):
        assert clock == self.NVML_CLOCK_SM
        return self.max_mhz

    def nvmlDeviceGetClockInfo(self, h, clock):
        return self.samples[min(self.i, len(self.samples) - 1)][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        r = self.samples[min(self.i, len(self.samples) - 1)][1]
        self.i += 1
        return r


class BrokenNvml(FakeNvml):
    def nvmlInit(self):
        raise RuntimeError("no NVML here")


def _run(sampler, seconds=0.15):
    sampler.start()
    time.sleep(seconds)
    return sampler.stop()


def test_nvml_samples_reasons_and_busy_median():
    # power cap while loaded, then idle samples (GPU idle bit, low clock)
    fake = FakeNvml([(1965, 0x0), (1400, 0x4), (1500, 0x4), (300, 0x1)])
    c = _run(bench.ClockSampler("GPU-0000", nvml=fake))
    assert c["source"] == "nvml"
    assert c["samples"] >= 4
    assert c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]
    # samples below half the maximum clock (idle) stay out of the median
    assert c["sm_mhz"] == 1500


def test_nvml_slowdown_reasons_are_named():
    fake = FakeNvml([(1200, 0x8 | 0x40), (1200, 0x20)])
    c = _run(bench.ClockSampler("0", nvml=fake))
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_fallback_when_nvml_does_not_start():
    c = _run(bench.ClockSampler("GPU-0000", nvml=BrokenNvml([])), seconds=0.05)
    # no GPU here: nvidia-smi is absent or answers nothing usable
    assert c is None or c["source"] == "nvidia-smi"
