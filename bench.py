#!/usr/bin/env python
"""Benchmark of the Step-3.5-Flash MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode] [--secondary prefill|none]

One step = one whole layer forward (router, top-k, counting sort, gather,
grouped gate|up GEMM + SwiGLU, grouped down GEMM, combine) over one batch of
T synthetic tokens, inputs already resident in HBM.  Weights are streamed
from HBM every step (touched experts: ~4 GB at T=64, ~6 GB at T=4096, far
larger than the 126 MB L2), so no L2 flush is needed between steps.

Multi-GPU (torchrun): every rank holds a replica of the layer and runs its own
batch (weak scaling, no collective on the data path); the step time is the
max over ranks.  Prints ONE JSON line on rank 0.

``--impl reference`` times the CPU fp64 oracle (the method's plain
definition) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at T=64 and T=4096; achieved fraction of HBM/TC roofline"


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode")
    ap.add_argument("--secondary",
                    default="prefill,zipf_prefill,clamp_ragged,tiny,decode_fp8,dense_decode,dense_prefill",
                    help="comma-separated further workloads measured in the same run")
    ap.add_argument("--parallel", choices=["auto", "ep", "replicas"], default="auto",
                    help="N > 1: expert parallelism (ep, the default: each rank holds 1/N of "
                         "the experts, all ranks route the same tokens, an NCCL all-reduce "
                         "sums the partial outputs) or independent replicas")
    ap.add_argument("--path", choices=["auto", "multi", "fused"], default="auto",
                    help="moe_forward's execution path (auto: the library's choice)")
    ap.add_argument("--detail", default="",
                    help="write the full record (per-stage times, every workload's rooflines) "
                         "to this JSON file; the printed line stays compact")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling case: override the token count T")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling case: override the number of routed experts "
                         "(smaller device footprint for ncu captures)")
    ap.add_argument("--intermediate", type=int, default=0,
                    help="profiling case: override the experts' intermediate size I (the "
                         "routing stages see the same inputs; smaller device footprint "
                         "for ncu captures of them)")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], tc_burst=d["bf16_tflops"],
                    tc_sustained=d.get("bf16_tflops_sustained") or d["bf16_tflops"],
                    source="measured")
    return dict(hbm=6650.0, tc_burst=1590.0, tc_sustained=1400.0, source="fallback")


# A timed region shorter than this runs at the burst clocks; a longer one
# settles at the power-capped sustained clocks.
SUSTAINED_REGION_MS = 1000.0


def _tc_peak(peaks, region_ms):
    """The bf16 tensor peak that applies to a timed region of region_ms:
    (TFLOP/s, label)."""
    if region_ms >= SUSTAINED_REGION_MS:
        return peaks["tc_sustained"], "sustained"
    return peaks["tc_burst"], "burst"


def _sig(v, n=4):
    """v rounded to n significant digits, as an int when that is whole (keeps
    the printed line short)."""
    if v is None or isinstance(v, (bool, int)) or v == 0:
        return v
    from math import floor, log10
    nd = n - 1 - int(floor(log10(abs(v))))
    r = round(v, nd)
    return int(r) if nd <= 0 else r


L2_BYTES = 126 * 1024 * 1024


def _config(wl, world):
    """The config dict both arms print (identical for the same workload)."""
    layer_bytes = (wl.num_experts + 1) * wl.weight_bytes_per_expert
    l2 = ("inputs > L2: weights streamed from HBM each step" if layer_bytes > L2_BYTES else
          "L2-resident: the whole layer fits in L2 (launch latency, not a roofline case)")
    return {"workload": wl.name, "T": wl.T, "hidden": wl.hidden, "experts": wl.num_experts,
            "top_k": wl.top_k, "intermediate": wl.intermediate, "shared_experts": 1,
            "parallelism": f"replicas x{world} (weak)", "l2": l2}


def _dtype(wl) -> str:
    """The arithmetic type of the expert GEMMs: fp32 weights take the fp32
    expert path (tf32 tensor cores over a two-term split, fp32-level
    results); bf16 and FP8 weights multiply in bf16."""
    return "f32" if wl.weight_dtype == "f32" else "bf16"


def _traffic_record(kernel: str, workload: str, groups: int, rows: int = 0):
    """ncu DRAM bytes per launch of `kernel`: the committed per-group figure
    times the launch's groups, plus (where the record has one) the per-row
    figure times the launch's token rows; None once the kernel's sources have
    changed since the capture."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    try:
        for line in open(p):
            f = line.split()
            if not f or f[0].startswith("#") or f[0] != f"{kernel}:{workload}":
                continue
            # the kernel's sources, comma-separated: their bytes hashed in order
            h = hashlib.sha256()
            for src in f[1].split(","):
                h.update(open(os.path.join(ROOT, src), "rb").read())
            if h.hexdigest() != f[2]:
                return None
            return int(f[3]) * groups + (int(f[4]) * rows if len(f) > 4 else 0)
    except Exception:
        return None
    return None


class ClockSampler:
    """SM clock and throttle-reason sampling around the timed region.  NVML
    (read-only queries) in a background thread every 10 ms; the nvidia-smi
    ``-lms`` loop is the fallback (its first sample comes only after its
    start-up, so a short region may get one or none).  ``stop()`` returns
    None when neither source gave a sample."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                   ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    PERIOD_S = 0.01

    def __init__(self, gpu_index, nvml=None):
        self.idx = gpu_index
        self.proc = None
        self._nvml = nvml          # a module with the pynvml interface (tests pass a fake)
        self._thread = None
        self._stop = None
        self._samples = []         # (sm MHz, reason bits)
        self._max = None

    def _start_nvml(self) -> bool:
        import threading
        try:
            nv = self._nvml
            if nv is None:
                import pynvml as nv
            nv.nvmlInit()
            if str(self.idx).startswith("GPU-"):
                h = nv.nvmlDeviceGetHandleByUUID(str(self.idx))
            else:
                h = nv.nvmlDeviceGetHandleByIndex(int(self.idx))
            self._max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            # one trial sample: an NVML without these queries falls back now
            self._samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                  int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
        except Exception:
            self._samples = []
            return False
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self._samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                          int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                except Exception:
                    pass
                self._stop.wait(self.PERIOD_S)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return True

    def start(self):
        if self._start_nvml():
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    @staticmethod
    def _summary(sm, mx, reasons, source):
        if not sm:
            return None
        busy = [v for v in sm if mx is None or v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": source}

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            reasons = {n for n, bit in self.REASON_BITS for _, r in self._samples if r & bit}
            return self._summary([v for v, _ in self._samples], self._max, reasons, "nvml")
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = [n for n, _ in self.REASON_BITS]
        for line in out.splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return self._summary(sm, mx, reasons, "nvidia-smi")


# ---------------------------------------------------------------- CPU oracle arm

def _oracle_sample(wl, x_host, rw, rb, experts, rows):
    import oracle.moe_oracle as om
    t0 = time.perf_counter()
    om.moe_forward_rows(rows, x_host, rw, rb, experts["w_gate"], experts["w_up"],
                        experts["w_down"], experts["sh_gate"], experts["sh_up"],
                        experts["sh_down"], top_k=wl.top_k, scale=wl.scale,
                        swiglu_limit=wl.swiglu_limit, swiglu_limit_shared=wl.swiglu_limit_shared)
    return time.perf_counter() - t0


class _PrefetchedExperts:
    """Host fp32 copies of the experts a sample touches (inputs in RAM before timing)."""

    def __init__(self, fetch, ids):
        self.m = {e: fetch(e) for e in ids}

    def __getitem__(self, e):
        return self.m[e]


def _sample_inputs_host(wl, x_host, rw, rb, rows, fetch_expert, shared):
    import oracle.moe_oracle as om
    r = om.moe_routing(x_host[rows], rw, rb, top_k=wl.top_k, scale=wl.scale)
    ids = sorted(set(int(e) for e in r["topk_idx"].reshape(-1)))
    got = {e: fetch_expert(e) for e in ids}
    experts = dict(w_gate=_PrefetchedExperts(lambda e: got[e][0], ids),
                   w_up=_PrefetchedExperts(lambda e: got[e][1], ids),
                   w_down=_PrefetchedExperts(lambda e: got[e][2], ids),
                   sh_gate=shared[0], sh_up=shared[1], sh_down=shared[2])
    return experts, len(ids)


def _arm_config(wl, world: int, parallel: str):
    """(config, scaling) of a line: both arms print the same for the same
    workload and GPU count (expert parallelism for N > 1 unless replicas are
    asked for, strong scaling; else replicas, weak scaling)."""
    if world > 1 and parallel != "replicas":
        return ep_config(wl, world), "strong"
    return _config(wl, world), "weak"


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import torch
    from sparse_moe_layer_gemm_b200.workloads import (WORKLOADS, draw_expert, draw_router,
                                                      draw_shared, draw_x)
    wl = WORKLOADS[a.workload]
    cores = len(os.sched_getaffinity(0))
    x = draw_x(wl, "cpu").float().numpy()
    rw, rb = (t.float().numpy() for t in draw_router(wl, "cpu"))
    sample = 1 if wl.hidden >= 4096 else wl.T
    rows = np.arange(sample)

    def fetch(e):
        return tuple(t.float().numpy() for t in draw_expert(wl, e, "cpu"))
    shared = tuple(t.float().numpy() for t in draw_shared(wl, "cpu"))
    experts, touched = _sample_inputs_host(wl, x, rw, rb, rows, fetch, shared)
    for _ in range(a.warmup):
        _oracle_sample(wl, x, rw, rb, experts, rows)
    secs = [_oracle_sample(wl, x, rw, rb, experts, rows) for _ in range(a.steps)]
    total = sum(secs)
    value = sample * a.steps / total
    config, scaling = _arm_config(wl, int(os.environ.get("WORLD_SIZE", a.gpus)), a.parallel)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": 1e3 * total / a.steps, "higher_is_better": True, "scaling": scaling,
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{sample} of {wl.T} tokens per step ({touched} routed experts "
                                   f"+ shared, weights drawn on the host, in RAM before timing)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def _measure(layer, x, steps, warmup, stream, record_stages=True):
    """Times exactly `steps` forwards (after `warmup`) with CUDA events on the
    launching stream; returns (ms per step, per-stage ms per step)."""
    import torch
    from sparse_moe_layer_gemm_b200 import binding as B
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            layer.forward(x)
        torch.cuda.synchronize()
        if record_stages:
            B.moe_set_stage_timing(layer.handle, steps)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            layer.forward(x)
        t1.record(stream)
        torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    stages = None
    if record_stages:
        tot, n = B.moe_get_stage_times(layer.handle)
        stages = {k: v / max(n, 1) for k, v in tot.items()}
        B.moe_set_stage_timing(layer.handle, 0)
    return ms, stages


def _routing_stats(layer, x):
    import torch
    out, rt = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    counts = rt["counts"].cpu()
    return int((counts > 0).sum()), int(counts.max())


def _kernel_roofline(wl, touched, stages_ms, peaks, ms_step, steps, fused=False):
    """Roofline of the dominant kernel and of the whole layer.  Multi-launch
    path: K5 gate|up, timed by its stage events.  Fused path: the one kernel
    is the whole layer (its time is stage 0).  The tensor peak is the burst
    figure for timed regions under a second (the kernel at its burst clocks),
    the sustained one for longer regions."""
    from sparse_moe_layer_gemm_b200.roofline import (algorithmic_bytes, algorithmic_flops,
                                                     gate_up_bytes, gate_up_flops)
    tc, tc_kind = _tc_peak(peaks, ms_step * steps)
    if fused:
        k_ms = stages_ms["router"]
        k_bytes = algorithmic_bytes(wl, touched)
        k_flops = algorithmic_flops(wl)
        kname = "moe_fused_kernel (whole layer)"
        trec = _traffic_record("fused", wl.name, touched + 1)
    else:
        k_ms = stages_ms["gate_up"]
        k_bytes = gate_up_bytes(wl, touched)
        k_flops = gate_up_flops(wl)
        # from 2048 tokens the library runs the expert GEMMs on CTA pairs
        # (FP8 weights: one-SM tiles with converter warps at every size)
        if wl.weight_dtype == "fp8":
            kname = "K5 gate_up fp8"
        else:
            kname = "K5 gate_up pairs" if wl.T >= 2048 else "K5 gate_up"
        # token rows of the launch: every routed copy plus the shared expert's
        trec = _traffic_record("gate_up", wl.name, touched + 1, wl.T * (wl.top_k + 1))
    t_bytes = k_bytes / (peaks["hbm"] * 1e9)
    t_flops = k_flops / (tc * 1e12)
    if t_bytes >= t_flops:
        ach = k_bytes / (k_ms * 1e-3) / 1e9
        rl = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
              "frac": ach / peaks["hbm"]}
    else:
        ach = k_flops / (k_ms * 1e-3) / 1e12
        rl = {"bound": "tensor", "achieved": ach, "peak": tc, "unit": "TFLOP/s",
              "frac": ach / tc}
    rl.update({"kernel": kname, "kernel_ms": k_ms,
               "algorithmic_bytes": k_bytes, "algorithmic_flops": k_flops,
               "peak_source": f"{peaks['source']}: hbm_gbs, bf16 {tc_kind}",
               "traffic": trec})
    lb = algorithmic_bytes(wl, touched)
    lf = algorithmic_flops(wl)
    t_layer = max(lb / (peaks["hbm"] * 1e9), lf / (tc * 1e12))
    layer = {"bound": "hbm" if lb / peaks["hbm"] >= lf / (tc * 1e3) else "tensor",
             "roofline_ms": 1e3 * t_layer, "frac": 1e3 * t_layer / ms_step,
             "bytes": lb, "flops": lf, "touched_experts": touched, "tensor_peak": tc_kind}
    return rl, layer


def _compact_roofline(rl):
    """The roofline object of the printed line (the contract's keys, short)."""
    out = {k: _sig(rl[k]) if isinstance(rl[k], float) else rl[k]
           for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    out["kernel"] = rl.get("kernel", rl.get("scope", ""))
    if "kernel_ms" in rl:
        out["kernel_ms"] = _sig(rl["kernel_ms"])
    return out


def _dense_secondary(wl, a, dev, world, rank, stream, peaks):
    """Times the dense SwiGLU MLP layer (K5 + K6 with one group of all T
    rows) on its own seeded inputs; roofline of the whole layer (HBM bytes of
    the weights + x + out, or flops on the sustained bf16 peak)."""
    import torch
    from sparse_moe_layer_gemm_b200 import binding as B
    from sparse_moe_layer_gemm_b200.replicas import job_throughput, max_over_ranks
    from sparse_moe_layer_gemm_b200.workloads import make_dense_inputs
    from dataclasses import replace as _replace
    inp = make_dense_inputs(_replace(wl, seed=wl.seed + rank), dev)
    layer = B.DenseMLP.from_workload(wl)
    layer.load_inputs(inp)
    x = inp["x"]
    steps, warm = a.steps, max(3, a.warmup)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            layer.forward(x)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            layer.forward(x)
        t1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    if layer.device_error() != 0:
        raise RuntimeError(f"device status word ({wl.name})")
    el_w = 2 if wl.weight_dtype == "bf16" else 4
    el_x = 2 if wl.act_dtype == "bf16" else 4
    H, I, T = wl.hidden, wl.intermediate, wl.T
    nbytes = 3 * H * I * el_w + 2 * T * H * el_x
    flops = 6 * T * H * I
    tc, tc_kind = _tc_peak(peaks, ms * steps)
    t_b, t_f = nbytes / (peaks["hbm"] * 1e9), flops / (tc * 1e12)
    if t_b >= t_f:
        rl = {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peaks["hbm"],
              "unit": "GB/s"}
    else:
        rl = {"bound": "tensor", "achieved": flops / (ms * 1e-3) / 1e12, "peak": tc,
              "unit": "TFLOP/s"}
    rl["frac"] = rl["achieved"] / rl["peak"]
    # up to 128 tokens the layer is one kernel (dense_streamk_kernel): its
    # committed ncu DRAM bytes per launch, while its sources are unchanged
    traffic = _traffic_record("dense", wl.name, 1) if T <= 128 else None
    rl.update({"scope": "whole dense layer (gate|up + down GEMMs)", "algorithmic_bytes": nbytes,
               "algorithmic_flops": flops, "traffic": traffic,
               "peak_source": f"{peaks['source']}: hbm_gbs, bf16 {tc_kind}"})
    layer.close()
    del inp, x
    torch.cuda.empty_cache()
    return {"workload": wl.name, "T": T, "value": job_throughput(T, world, ms), "unit": "tokens/s",
            "ms_per_step": ms, "roofline": rl, "layer_roofline": {"frac": rl["frac"],
                                                                  "bound": rl["bound"]},
            "layer": f"dense SwiGLU MLP, H={H}, I={I} (the first three decoder layers)"}


def run_ours(a):
    import torch
    import torch.distributed as dist
    from sparse_moe_layer_gemm_b200 import binding as B
    from sparse_moe_layer_gemm_b200.replicas import (job_throughput, max_over_ranks,
                                                     rank_batch_workload)
    from sparse_moe_layer_gemm_b200.workloads import (DENSE_WORKLOADS, WORKLOADS, draw_x,
                                                      make_inputs)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B.load_library()
    wl = WORKLOADS[a.workload]
    if a.experts or a.tokens or a.intermediate:
        from dataclasses import replace as _replace
        I = a.intermediate or wl.intermediate
        Is = a.intermediate or wl.shared_intermediate
        wl = _replace(wl, num_experts=a.experts or wl.num_experts, T=a.tokens or wl.T,
                      intermediate=I, shared_intermediate=Is,
                      name=f"{wl.name}_e{a.experts or wl.num_experts}_t{a.tokens or wl.T}"
                           + (f"_i{I}" if a.intermediate else ""))
    peaks = _peaks()

    inp = make_inputs(wl, dev)                          # weights replicated on every rank
    x = draw_x(rank_batch_workload(wl, rank), dev)      # each rank its own batch
    layer = B.MoeLayer.from_workload(wl)
    path = {"auto": B.MOE_PATH_AUTO, "multi": B.MOE_PATH_MULTI, "fused": B.MOE_PATH_FUSED}[a.path]
    layer.set_path(path)
    layer.load_inputs(inp)
    stream = torch.cuda.Stream(device=dev)
    touched, max_rows = _routing_stats(layer, x)

    def barrier():
        if world > 1:
            dist.barrier()

    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
    except Exception:
        gpu_id = str(local)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(a.warmup):
            layer.forward(x)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms, _ = _measure(layer, x, a.steps, 0, stream, record_stages=False)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(ms, dev)
    # per-stage durations (and the dominant kernel's) from a second pass of
    # the same K steps with CUDA events between the kernels; kept out of the
    # timed region above because the events themselves cost ~4 % at T=64
    _, stages = _measure(layer, x, a.steps, 0, stream, record_stages=True)
    err = layer.device_error()
    if err != 0:
        raise RuntimeError(f"device status word {err}")
    value = job_throughput(wl.T, world, ms)
    fused = B.moe_forward_path(layer.handle, wl.T) == B.MOE_PATH_FUSED
    kr, lr = _kernel_roofline(wl, touched, stages, peaks, ms, a.steps, fused)

    e2e = None
    if not a.no_e2e:
        # every step copies its input from pinned host memory and its result
        # back: the pipelined entry point (moe_forward_host_async: a step's
        # copies overlap its neighbours' forwards), and, for comparison, the
        # synchronous one (moe_forward_host: copy, forward, copy, wait)
        xh = x.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        n = a.steps

        def timed(step, finish):
            with torch.cuda.stream(stream):
                for _ in range(max(1, a.warmup)):
                    step()
                finish()
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(n):
                    step()
                finish()
                e1.record(stream)
                torch.cuda.synchronize()
            return max_over_ranks(e0.elapsed_time(e1) / n, dev)

        et = timed(lambda: layer.forward_host_async(xh, oh, stream=stream),
                   lambda: layer.forward_host_join(stream=stream))
        et_sync = timed(lambda: layer.forward_host(xh, oh, stream=stream), lambda: None)
        el = 2 if wl.act_dtype == "bf16" else 4
        e2e = {"value": job_throughput(wl.T, world, et), "unit": "tokens/s",
               "sync_value": job_throughput(wl.T, world, et_sync),
               "h2d_bytes_per_step": wl.T * wl.hidden * el,
               "d2h_bytes_per_step": wl.T * wl.hidden * el,
               "path": "moe_forward_host_async (pinned host x/out; every step's input and "
                       "result copies inside the timed region, overlapped with the "
                       "neighbouring steps' forwards); sync_value: moe_forward_host "
                       "(copy, forward, copy, wait per step)"}

    secondary = []
    for name2 in [n for n in (a.secondary or "").split(",") if n and n != "none" and n != a.workload]:
        if name2 in DENSE_WORKLOADS:  # the dense MLP layer (no routing)
            barrier()
            secondary.append(_dense_secondary(DENSE_WORKLOADS[name2], a, dev, world, rank, stream,
                                              peaks))
            continue
        wl2 = WORKLOADS[name2]
        same_experts = (wl2.expert_std == wl.expert_std and wl2.weight_dtype == wl.weight_dtype
                        and wl2.hidden == wl.hidden and wl2.num_experts == wl.num_experts
                        and wl2.swiglu_limit == wl.swiglu_limit)
        layer2, inp2 = layer, None
        if not same_experts:  # its own layer and weights (clamped / tiny configs)
            inp2 = make_inputs(wl2, dev)
            layer2 = B.MoeLayer.from_workload(wl2)
            layer2.set_path(path)
            layer2.load_inputs(inp2)
        elif wl2.bias != wl.bias:  # same experts, another router bias
            from sparse_moe_layer_gemm_b200.workloads import draw_router
            _, rb2 = draw_router(wl2, dev)
            layer.load_weights(inp["router_w"], rb2, inp["w_gate"], inp["w_up"], inp["w_down"],
                               inp["sh_gate"], inp["sh_up"], inp["sh_down"])
        x2 = draw_x(rank_batch_workload(wl2, rank), dev)
        touched2, _ = _routing_stats(layer2, x2)
        barrier()
        ms2, _ = _measure(layer2, x2, a.steps, max(3, a.warmup), stream, record_stages=False)
        ms2 = max_over_ranks(ms2, dev)
        _, st2 = _measure(layer2, x2, a.steps, 0, stream)
        if layer2.device_error() != 0:
            raise RuntimeError(f"device status word {layer2.device_error()} ({wl2.name})")
        fused2 = B.moe_forward_path(layer2.handle, wl2.T) == B.MOE_PATH_FUSED
        kr2, lr2 = _kernel_roofline(wl2, touched2, st2, peaks, ms2, a.steps, fused2)
        entry = {"workload": wl2.name, "T": wl2.T, "value": job_throughput(wl2.T, world, ms2),
                 "unit": "tokens/s", "ms_per_step": ms2, "roofline": kr2,
                 "layer_roofline": lr2, "stage_ms": st2,
                 "path": "fused" if fused2 else "multi-launch"}
        if wl2.weight_dtype != "bf16":
            entry["weights"] = {"fp8": "fp8_e4m3 codes + fp32 per-feature scales (bf16 MMA)",
                                "f32": "fp32: tf32 tensor cores over a two-term split of "
                                       "every operand (fp32 expert path)"}[wl2.weight_dtype]
        if wl2.name == "tiny":
            entry["l2"] = "L2-resident (16 KB experts): launch latency, not a roofline case"
        secondary.append(entry)
        del x2
        if inp2 is not None:
            layer2.close()
            del inp2
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = _cpu_baseline_from_device(wl, inp, x)

    launches = B.moe_kernel_launches(layer.handle, wl.T) * a.steps
    if rank == 0:
        full = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": _dtype(wl), "data": "synthetic",
            "config": _config(wl, world), "roofline": kr, "layer_roofline": lr,
            "stage_ms": stages,
            "routing": {"touched_experts": touched, "max_rows_per_expert": max_rows},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
            "secondary": secondary,
        }
        if a.detail:
            with open(a.detail, "w") as f:
                json.dump(full, f, indent=1)
        print(json.dumps(_compact_line(full), separators=(",", ":")), flush=True)
    layer.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def ep_plan(num_experts: int, world: int, rank: int) -> dict:
    """This rank's part of the expert-parallel layer: its contiguous shard of
    the routed experts and whether it holds the shared expert."""
    from sparse_moe_layer_gemm_b200.expert_parallel import holds_shared, shard_range
    first, count = shard_range(num_experts, world, rank)
    return {"first": first, "count": count, "with_shared": holds_shared(rank)}


def ep_config(wl, world: int) -> dict:
    cfg = _config(wl, world)
    cfg["parallelism"] = f"ep{world}: experts sharded, all-reduce of the partial outputs"
    return cfg


def run_ep(a):
    """N > 1, expert parallelism: every rank routes the same T tokens over all
    experts, computes the pairs of its own shard (rank 0 also the shared
    expert) and an NCCL all-reduce sums the bf16 partial outputs; each rank
    draws and loads only its shard's expert tensors.  One step = the forward
    plus the all-reduce; the job processes T tokens per step (strong scaling:
    the work per step is fixed, the experts per GPU shrink with N)."""
    import datetime
    import torch
    import torch.distributed as dist
    from sparse_moe_layer_gemm_b200 import binding as B
    from sparse_moe_layer_gemm_b200.replicas import max_over_ranks
    from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, draw_router, draw_x, \
        make_shard_inputs

    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    B.load_library()
    peaks = _peaks()
    stream = torch.cuda.Stream(device=dev)
    path = {"auto": B.MOE_PATH_AUTO, "multi": B.MOE_PATH_MULTI, "fused": B.MOE_PATH_FUSED}[a.path]

    def step(layer, x, out):
        layer.forward(x, out)
        dist.all_reduce(out, op=dist.ReduceOp.SUM)

    def timed(layer, x, out, steps, warmup):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                step(layer, x, out)
            torch.cuda.synchronize()
            dist.barrier()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                step(layer, x, out)
            e1.record(stream)
            torch.cuda.synchronize()
        dist.barrier()
        return max_over_ranks(e0.elapsed_time(e1) / steps, dev)

    def measure(wl, layer, inp):
        x = inp["x"]
        out = torch.empty_like(x)
        _, rt = layer.forward(x, routing=True)
        torch.cuda.synchronize()
        touched_local = int((rt["counts"][:plan["count"]] > 0).sum())  # the shard's experts
        t = torch.tensor([touched_local], device=dev)
        dist.all_reduce(t)                     # routed experts touched by the whole job
        ms = timed(layer, x, out, a.steps, a.warmup)
        B.moe_set_stage_timing(layer.handle, a.steps)
        with torch.cuda.stream(stream):
            for _ in range(a.steps):
                layer.forward(x, out)
        torch.cuda.synchronize()
        tot, n = B.moe_get_stage_times(layer.handle)
        B.moe_set_stage_timing(layer.handle, 0)
        stages = {k: v / max(n, 1) for k, v in tot.items()}
        if layer.device_error() != 0:
            raise RuntimeError(f"device status word ({wl.name})")
        fused = B.moe_forward_path(layer.handle, wl.T) == B.MOE_PATH_FUSED
        # the dominant kernel on this rank (its own touched experts); the
        # layer against the whole job's HBM bandwidth (N GPUs)
        kr, _ = _kernel_roofline(wl, touched_local, stages, peaks, ms, a.steps, fused)
        job = dict(peaks, hbm=peaks["hbm"] * world, tc_burst=peaks["tc_burst"] * world,
                   tc_sustained=peaks["tc_sustained"] * world)
        _, lr = _kernel_roofline(wl, int(t.item()), stages, job, ms, a.steps, fused)
        return ms, stages, kr, lr, x, out

    wl = WORKLOADS[a.workload]
    plan = ep_plan(wl.num_experts, world, rank)
    shard = (plan["first"], plan["count"], 1 if plan["with_shared"] else 0)
    inp = make_shard_inputs(wl, plan["first"], plan["count"], plan["with_shared"], dev)
    layer = B.MoeLayer.from_workload(wl, shard)
    layer.set_path(path)
    layer.load_shard_weights(inp["router_w"], inp["router_bias"], inp["w_gate"], inp["w_up"],
                             inp["w_down"], inp.get("sh_gate"), inp.get("sh_up"),
                             inp.get("sh_down"))
    sampler = ClockSampler(str(local))
    sampler.start()
    ms, stages, kr, lr, x, out = measure(wl, layer, inp)
    clocks = sampler.stop()
    value = wl.T / (ms * 1e-3)

    e2e = None
    if not a.no_e2e:
        xh = x.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        xd = torch.empty_like(x)
        with torch.cuda.stream(stream):
            for _ in range(max(1, a.warmup)):
                xd.copy_(xh, non_blocking=True)
                step(layer, xd, out)
                oh.copy_(out, non_blocking=True)
            torch.cuda.synchronize()
            dist.barrier()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(a.steps):
                xd.copy_(xh, non_blocking=True)
                step(layer, xd, out)
                oh.copy_(out, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize()
        et = max_over_ranks(e0.elapsed_time(e1) / a.steps, dev)
        io = wl.T * wl.hidden * (2 if wl.act_dtype == "bf16" else 4)
        e2e = {"value": wl.T / (et * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": world * io, "d2h_bytes_per_step": world * io,
               "path": "every rank: pinned x in, forward + all-reduce, out back to the host"}

    secondary = []
    for name2 in [n for n in (a.secondary or "").split(",") if n and n != "none"]:
        if name2 not in ("prefill", "zipf_prefill") or name2 == a.workload:
            continue  # the same experts, another batch and router bias
        wl2 = WORKLOADS[name2]
        _, rb2 = draw_router(wl2, dev)
        layer.load_shard_weights(inp["router_w"], rb2, inp["w_gate"], inp["w_up"], inp["w_down"],
                                 inp.get("sh_gate"), inp.get("sh_up"), inp.get("sh_down"))
        inp2 = dict(inp, x=draw_x(wl2, dev))
        ms2, st2, kr2, lr2, _, _ = measure(wl2, layer, inp2)
        secondary.append({"workload": wl2.name, "T": wl2.T, "value": wl2.T / (ms2 * 1e-3),
                          "unit": "tokens/s", "ms_per_step": ms2, "roofline": kr2,
                          "layer_roofline": lr2, "stage_ms": st2})
        del inp2
    launches = B.moe_kernel_launches(layer.handle, wl.T) * a.steps
    if rank == 0:
        full = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": _dtype(wl), "data": "synthetic",
            "config": ep_config(wl, world), "roofline": kr, "layer_roofline": lr,
            "stage_ms": stages, "routing": {}, "cpu_baseline": None, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks, "secondary": secondary,
        }
        if a.detail:
            with open(a.detail, "w") as f:
                json.dump(full, f, indent=1)
        print(json.dumps(_compact_line(full), separators=(",", ":")), flush=True)
    layer.close()
    dist.barrier()
    dist.destroy_process_group()
    return 0


def _compact_line(full):
    """The one printed JSON line, kept under 1500 characters: the contract's
    keys with short values, the headline's layer roofline fraction, then the
    other workloads as [tokens/s, layer roofline fraction] and, last, the
    prefill (T=4096) half of the metric in full; per-stage tables and every
    workload's kernel rooflines stay in the --detail file."""
    line = {k: full[k] for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup",
                                 "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                                 "dtype", "data", "config")}
    line["value"] = _sig(line["value"], 6)
    line["ms_per_step"] = _sig(line["ms_per_step"], 5)
    line["roofline"] = _compact_roofline(full["roofline"])
    line["layer_roofline"] = {"bound": full["layer_roofline"]["bound"],
                              "frac": _sig(full["layer_roofline"]["frac"])}
    cpu = full["cpu_baseline"]
    if cpu is not None:
        cpu = {"value": _sig(cpu["value"]), "unit": cpu["unit"], "cores": cpu["cores"],
               "kind": cpu["kind"], "sample": cpu["short"]}
    line["cpu_baseline"] = cpu
    e2e = full["e2e"]
    if e2e is not None:
        e2e = {k: (_sig(v, 6) if k in ("value", "sync_value") else v) for k, v in e2e.items()
               if k != "path"}
    line["e2e"] = e2e
    line["gpu_launches"] = full["gpu_launches"]
    c = full["clocks"]
    line["clocks"] = None if c is None else {"sm_mhz": c["sm_mhz"], "sm_max_mhz": c["sm_max_mhz"],
                                             "reasons": c["reasons"]}
    others, pre = {}, None
    for e in full["secondary"]:
        if e["workload"] == "prefill" and pre is None:
            pre = {"T": e["T"], "value": _sig(e["value"], 6),
                   "ms_per_step": _sig(e["ms_per_step"], 5),
                   "layer_roofline": {"bound": e["layer_roofline"]["bound"],
                                      "frac": _sig(e["layer_roofline"]["frac"])},
                   "roofline": _compact_roofline(e["roofline"])}
        else:
            others[e["workload"]] = [_sig(e["value"], 3), _sig(e["layer_roofline"]["frac"], 3)]
    line["others"] = others
    if pre is not None:
        line["prefill"] = pre
    return line


def _cpu_baseline_from_device(wl, inp, x):
    """The oracle on the host cores on a bounded sample of the same batch
    (weights copied from the device before timing)."""
    import numpy as np
    from sparse_moe_layer_gemm_b200.workloads import host_f32
    xh = host_f32(x)
    rw = host_f32(inp["router_w"])
    rb = host_f32(inp["router_bias"])
    sample = min(wl.T, 8)
    rows = np.arange(sample)

    def fetch(e):
        return (host_f32(inp["w_gate"][e]), host_f32(inp["w_up"][e]), host_f32(inp["w_down"][e]))
    shared = (host_f32(inp["sh_gate"]), host_f32(inp["sh_up"]), host_f32(inp["sh_down"]))
    experts, touched = _sample_inputs_host(wl, xh, rw, rb, rows, fetch, shared)
    secs = _oracle_sample(wl, xh, rw, rb, experts, rows)
    return {"value": sample / secs, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{sample} of {wl.T} tokens of the same batch, {touched} routed experts "
                      f"+ shared, fp64 NumPy, weights in host RAM before timing",
            "short": f"{sample}/{wl.T} tokens, {touched} experts + shared, fp64",
            "seconds": secs}


def main():
    a = _args()
    if a.impl == "reference":
        return run_reference(a)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and a.parallel != "replicas":
        return run_ep(a)
    return run_ours(a)


if __name__ == "__main__":
    sys.exit(main())
