"""bench.py host logic on the CPU: the clock sampler against a fake NVML
(the reasons it reports, the median over samples under load, the fallback
when NVML cannot start), the DRAM-traffic records (reported only while
the captured kernel's sources still hash as recorded), and the config and
dtype a line reports for its workload."""
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
    assert bench._traffic_record("gate_up", "decode", 33, rows=500) == 33000  # no row term
    assert bench._traffic_record("gate_up", "prefill", 33) is None      # no record
    with open(os.path.join(root, "k.cuh"), "ab") as f:                  # the kernel changes
        f.write(b" ")
    assert bench._traffic_record("gate_up", "decode", 33) is None


def test_traffic_record_row_term(tmp_path, monkeypatch):
    """A fifth column adds bytes per token row of the launch."""
    root = str(tmp_path)
    with open(os.path.join(root, "k.cu"), "wb") as f:
        f.write(b"kernel body")
    digest = hashlib.sha256(b"kernel body").hexdigest()
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "dram_traffic.txt"), "w") as f:
        f.write(f"gate_up:prefill k.cu {digest} 1000 7\n")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench._traffic_record("gate_up", "prefill", 10, rows=100) == 10 * 1000 + 100 * 7


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
        assert len(f) in (4, 5), line
        for src in f[1].split(","):
            assert os.path.exists(os.path.join(bench.ROOT, src)), src
        keys.append(f[0])
    assert keys, "no records"


def _fake_full(n_secondary=6):
    from sparse_moe_layer_gemm_b200.workloads import WORKLOADS
    peaks = bench._peaks()
    wl, wp = WORKLOADS["decode"], WORKLOADS["prefill"]
    kr, lr = bench._kernel_roofline(wl, 131, {"gate_up": 0.4021234}, peaks, 0.62099, 200)
    kr2, lr2 = bench._kernel_roofline(wp, 201, {"gate_up": 1.0712345}, peaks, 1.7131, 200)
    kr2["traffic"] = 4533671234
    sec = [{"workload": n, "T": 1, "value": 12345678.91, "ms_per_step": 1.0,
            "roofline": kr2, "layer_roofline": lr2}
           for n in ["zipf_prefill", "clamp_ragged", "tiny", "decode_fp8", "dense_decode",
                     "dense_prefill"][:n_secondary]]
    sec.insert(1, {"workload": "prefill", "T": 4096, "value": 2391694.123,
                   "ms_per_step": 1.7131234, "roofline": kr2, "layer_roofline": lr2})
    return {"metric": bench.METRIC, "value": 103059.849, "unit": "tokens/s", "n_gpus": 8,
            "steps": 200, "warmup": 5, "ms_per_step": 0.62099838, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench._config(wl, 8), "roofline": kr, "layer_roofline": lr,
            "stage_ms": {}, "routing": {},
            "cpu_baseline": {"value": 9.4835962, "unit": "tokens/s", "cores": 128,
                             "kind": "oracle", "short": "8/64 tokens, 148 experts + shared, fp64"},
            "e2e": {"value": 91327.955, "unit": "tokens/s", "h2d_bytes_per_step": 524288,
                    "d2h_bytes_per_step": 524288, "path": "p"},
            "gpu_launches": 1400,
            "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                       "reasons": ["sw_power_cap", "hw_slowdown"], "samples": 9,
                       "source": "nvml"},
            "secondary": sec}


def test_compact_line_fits_the_tail_and_ends_with_prefill():
    """The printed line stays under 1500 characters (the part of stdout the
    round's record keeps) and ends with the T=4096 half of the metric."""
    import json
    line = bench._compact_line(_fake_full())
    s = json.dumps(line, separators=(",", ":"))
    assert len(s) < 1500, len(s)
    assert list(line)[-1] == "prefill"
    pre = line["prefill"]
    assert pre["T"] == 4096 and pre["roofline"]["traffic"] == 4533671234
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in line["roofline"] and k in pre["roofline"]
    assert set(line["others"]) == {"zipf_prefill", "clamp_ragged", "tiny", "decode_fp8",
                                   "dense_decode", "dense_prefill"}


def test_tensor_peak_follows_the_timed_region():
    peaks = bench._peaks()
    assert bench._tc_peak(peaks, 999.0) == (peaks["tc_burst"], "burst")
    assert bench._tc_peak(peaks, 1000.0) == (peaks["tc_sustained"], "sustained")
    from sparse_moe_layer_gemm_b200.workloads import WORKLOADS
    wl = WORKLOADS["zipf_prefill"]
    # a 20-step region of 4 ms steps is short: burst peak
    kr, lr = bench._kernel_roofline(wl, 28, {"gate_up": 2.5}, peaks, 4.0, 20)
    assert kr["bound"] == "tensor" and kr["peak"] == peaks["tc_burst"]
    assert lr["tensor_peak"] == "burst"
    kr, lr = bench._kernel_roofline(wl, 28, {"gate_up": 2.5}, peaks, 4.0, 500)
    assert kr["peak"] == peaks["tc_sustained"] and lr["tensor_peak"] == "sustained"


def test_both_arms_print_the_same_config():
    from sparse_moe_layer_gemm_b200.workloads import WORKLOADS
    wl = WORKLOADS["decode"]
    assert bench._config(wl, 4) == _fake_full()["config"] or bench._config(wl, 8) == \
        _fake_full()["config"]


def test_config_and_dtype_follow_the_workload():
    """The printed config is identical for both arms of a workload; its L2
    note and the line's dtype follow the workload: the full layer streams its
    weights from HBM, the tiny fp32 layer fits in L2 and runs the fp32
    expert path."""
    from sparse_moe_layer_gemm_b200.workloads import WORKLOADS
    dec, tiny = WORKLOADS["decode"], WORKLOADS["tiny"]
    assert bench._config(dec, 1) == bench._config(dec, 1)
    assert bench._config(dec, 1)["l2"].startswith("inputs > L2")
    assert bench._config(tiny, 1)["l2"].startswith("L2-resident")
    assert bench._dtype(dec) == "bf16"
    assert bench._dtype(WORKLOADS["decode_fp8"]) == "bf16"   # the MMA is bf16 on the codes
    assert bench._dtype(tiny) == "f32"


def test_both_arms_print_the_same_config_at_every_gpu_count():
    """The reference arm's config and scaling are the ones our arm prints for
    the same workload and N: the full config at N = 1, expert parallelism
    (strong scaling) for N > 1 by default, replicas (weak) when asked."""
    from sparse_moe_layer_gemm_b200.workloads import WORKLOADS
    wl = WORKLOADS["decode"]
    assert bench._arm_config(wl, 1, "auto") == (bench._config(wl, 1), "weak")
    assert bench._arm_config(wl, 4, "auto") == (bench.ep_config(wl, 4), "strong")
    assert bench._arm_config(wl, 4, "ep") == (bench.ep_config(wl, 4), "strong")
    assert bench._arm_config(wl, 4, "replicas") == (bench._config(wl, 4), "weak")
