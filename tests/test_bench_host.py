"""bench.py host logic on the CPU: the clock sampler against a fake NVML
(the reasons it reports, the median over samples under load, the fallback
when NVML cannot start) and the DRAM-traffic records (reported only while
the captured kernel's sources still hash as recorded)."""
import hashlib
import os
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


def _write_record(root, sources, digest, per_group):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "dram_traffic.txt"), "w") as f:
        f.write("# key sources sha256 bytes_per_group\n")
        f.write(f"gate_up:decode {','.join(sources)} {digest} {per_group}\n")


def test_traffic_record_follows_the_source_hash(tmp_path, monkeypatch):
    root = str(tmp_path)
    srcs = ["k.cu", "k.cuh"]
    for name, body in zip(srcs, (b"kernel body", b"header body")):
        with open(os.path.join(root, name), "wb") as f:
            f.write(body)
    h = hashlib.sha256()
    h.update(b"kernel body")
    h.update(b"header body")
    _write_record(root, srcs, h.hexdigest(), 1000)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench._traffic_record("gate_up", "decode", 33) == 33000
    assert bench._traffic_record("gate_up", "prefill", 33) is None      # no record
    with open(os.path.join(root, "k.cuh"), "ab") as f:                  # the kernel changes
        f.write(b" ")
    assert bench._traffic_record("gate_up", "decode", 33) is None


def test_committed_traffic_records_match_the_sources():
    """Every committed record names sources that exist; the bench reports a
    record's traffic only while their hash matches, so a stale record shows
    as null rather than as a number for another kernel."""
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic.txt")
    keys = []
    for line in open(path):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        assert len(f) == 4, line
        for src in f[1].split(","):
            assert os.path.exists(os.path.join(bench.ROOT, src)), src
        keys.append(f[0])
    assert keys, "no records"
