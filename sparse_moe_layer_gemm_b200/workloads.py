"""Seeded synthetic workloads for the Step-3.5-Flash MoE FFN layer.

This module only draws inputs; it holds none of the layer's arithmetic and
loads no native code, so both the CUDA path and the CPU oracle can be fed from
it.  The shapes follow the layer's configuration (llm-atlas "Step-3.5-Flash",
table "Raw config fields": hidden 4096, 288 routed experts, top-8,
moe_intermediate_size 1280, share_expert_dim 1280, swiglu_limits 7); the value
distributions are synthetic stand-ins for real activations and trained weights,
which the pages do not provide.

Every tensor is drawn from its own torch generator, seeded from
(seed, stream id), so any one expert can be regenerated alone.  Small
workloads are drawn on the CPU; full-size ones (9 GB of expert weights) are
drawn on the device with torch's CUDA generator and copied to the host piece
by piece for the oracle.  The two devices give different (but each
deterministic) values; a test always hands the same tensors to both sides.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    hidden: int
    num_experts: int
    top_k: int
    intermediate: int
    shared_intermediate: int
    act_dtype: str                 # "f32" or "bf16"
    weight_dtype: str              # "f32", "bf16" or "fp8" (E4M3 codes + scales)
    x_dist: str                    # "normal" or "rmsnorm_normal"
    router_std: float
    expert_std: float
    bias: str                      # "normal0.1", "zipf" or "zero"
    swiglu_limit: float = 0.0
    swiglu_limit_shared: float = 0.0
    scale: float = 3.0
    seed: int = 0
    description: str = ""

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T)

    @property
    def weight_bytes_per_expert(self) -> int:
        el = {"fp8": 1, "bf16": 2, "f32": 4}[self.weight_dtype]
        return 3 * self.hidden * self.intermediate * el


_STEP35 = dict(hidden=4096, num_experts=288, top_k=8, intermediate=1280,
               shared_intermediate=1280, act_dtype="bf16", weight_dtype="bf16",
               x_dist="rmsnorm_normal", router_std=0.02)

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(
        name="tiny", T=32, hidden=256, num_experts=16, top_k=4, intermediate=64,
        shared_intermediate=64, act_dtype="f32", weight_dtype="f32",
        x_dist="normal", router_std=0.02, expert_std=0.05, bias="normal0.1",
        description="T=32, H=256, 16 experts top-4 + shared, I=64, fp32"),
    "decode": Workload(
        name="decode", T=64, expert_std=0.02, bias="normal0.1",
        description="Step-3.5-Flash MoE layer, decode shape T=64", **_STEP35),
    "prefill": Workload(
        name="prefill", T=4096, expert_std=0.02, bias="normal0.1",
        description="Step-3.5-Flash MoE layer, prefill shape T=4096", **_STEP35),
    "zipf_prefill": Workload(
        name="zipf_prefill", T=16384, expert_std=0.02, bias="zipf",
        description="load-imbalanced prefill T=16384, Zipf router bias", **_STEP35),
    "decode_fp8": Workload(
        name="decode_fp8", T=64, expert_std=0.02, bias="normal0.1",
        description="decode shape T=64 with FP8 E4M3 expert weights (per-feature scales)",
        **dict(_STEP35, weight_dtype="fp8")),
    "prefill_fp8": Workload(
        name="prefill_fp8", T=4096, expert_std=0.02, bias="normal0.1",
        description="prefill shape T=4096 with FP8 E4M3 expert weights (per-feature scales)",
        **dict(_STEP35, weight_dtype="fp8")),
    "clamp_ragged": Workload(
        name="clamp_ragged", T=3001, expert_std=0.05, bias="normal0.1",
        swiglu_limit=7.0, swiglu_limit_shared=7.0,
        description="clamped SwiGLU (limit 7), ragged T=3001", **_STEP35),
}

# stream ids of the per-tensor generators
_S_X, _S_ROUTER, _S_BIAS, _S_SHARED = 1, 2, 3, 10
_S_EXPERT = 1000


def _gen(device: torch.device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed << 24) + stream)
    return g


def _torch_dtype(name: str) -> torch.dtype:
    # fp8 weights are drawn in fp32, then quantised (quantize_e4m3)
    return {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float32}[name]


def quantize_e4m3(w: torch.Tensor):
    """Input preparation for FP8 weight workloads: ``w`` [..., K, N] (x @ W
    layout, N output features) -> (codes uint8 [..., K, N], scale fp32
    [..., N]).  Each output feature gets the power of two
    scale = 2^ceil(log2(amax / 448)) (1 for an all-zero feature), so w / scale
    lies within the E4M3FN range, and the codes are torch's round-to-nearest
    float8_e4m3fn conversion of w / scale."""
    wf = w.float()
    amax = wf.abs().amax(dim=-2)
    e = torch.ceil(torch.log2(torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))))
    scale = torch.exp2(e)
    codes = (wf / scale.unsqueeze(-2)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


def draw_x(wl: Workload, device="cpu") -> torch.Tensor:
    dev = torch.device(device)
    x = torch.randn(wl.T, wl.hidden, generator=_gen(dev, wl.seed, _S_X),
                    device=dev, dtype=torch.float32)
    if wl.x_dist == "rmsnorm_normal":
        # rows rescaled to unit root-mean-square (no epsilon, no weight)
        x = x / torch.sqrt(torch.mean(x * x, dim=1, keepdim=True))
    return x.to(_torch_dtype(wl.act_dtype))


def draw_router(wl: Workload, device="cpu"):
    dev = torch.device(device)
    w = torch.randn(wl.hidden, wl.num_experts, generator=_gen(dev, wl.seed, _S_ROUTER),
                    device=dev, dtype=torch.float32) * wl.router_std
    if wl.bias == "normal0.1":
        b = torch.randn(wl.num_experts, generator=_gen(dev, wl.seed, _S_BIAS),
                        device=dev, dtype=torch.float32) * 0.1
    elif wl.bias == "zipf":
        # b_e = 0.5 * ln(1 / (e+1)^1.1), e 0-based, natural log
        e = torch.arange(wl.num_experts, dtype=torch.float64)
        b = (-0.55 * torch.log(e + 1.0)).to(torch.float32).to(dev)
    elif wl.bias == "zero":
        b = torch.zeros(wl.num_experts, dtype=torch.float32, device=dev)
    else:
        raise ValueError(wl.bias)
    return w, b


def draw_expert(wl: Workload, e: int, device="cpu"):
    """Routed expert e: (w_gate [H, I], w_up [H, I], w_down [I, H])."""
    dev = torch.device(device)
    g = _gen(dev, wl.seed, _S_EXPERT + e)
    H, I = wl.hidden, wl.intermediate
    dt = _torch_dtype(wl.weight_dtype)
    wg = (torch.randn(H, I, generator=g, device=dev) * wl.expert_std).to(dt)
    wu = (torch.randn(H, I, generator=g, device=dev) * wl.expert_std).to(dt)
    wd = (torch.randn(I, H, generator=g, device=dev) * wl.expert_std).to(dt)
    return wg, wu, wd


def draw_shared(wl: Workload, device="cpu"):
    dev = torch.device(device)
    g = _gen(dev, wl.seed, _S_SHARED)
    H, I = wl.hidden, wl.shared_intermediate
    dt = _torch_dtype(wl.weight_dtype)
    wg = (torch.randn(H, I, generator=g, device=dev) * wl.expert_std).to(dt)
    wu = (torch.randn(H, I, generator=g, device=dev) * wl.expert_std).to(dt)
    wd = (torch.randn(I, H, generator=g, device=dev) * wl.expert_std).to(dt)
    return wg, wu, wd


def make_inputs(wl: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """All tensors of a workload, in the ABI's layouts:
    x [T, H]; router_w [H, E] f32; router_bias [E] f32;
    w_gate, w_up [E, H, I]; w_down [E, I, H]; sh_gate, sh_up [H, Is]; sh_down [Is, H].
    FP8 weights: the six weight tensors hold E4M3FN codes (uint8) and
    s_w_gate, s_w_up [E, I], s_w_down [E, H], s_sh_gate, s_sh_up [Is],
    s_sh_down [H] their per-output-feature scales (fp32)."""
    dev = torch.device(device)
    x = draw_x(wl, dev)
    rw, rb = draw_router(wl, dev)
    E, H, I = wl.num_experts, wl.hidden, wl.intermediate
    dt = _torch_dtype(wl.weight_dtype)
    w_gate = torch.empty(E, H, I, dtype=dt, device=dev)
    w_up = torch.empty(E, H, I, dtype=dt, device=dev)
    w_down = torch.empty(E, I, H, dtype=dt, device=dev)
    for e in range(E):
        wg, wu, wd = draw_expert(wl, e, dev)
        w_gate[e].copy_(wg)
        w_up[e].copy_(wu)
        w_down[e].copy_(wd)
    sg, su, sd = draw_shared(wl, dev)
    out = dict(x=x, router_w=rw, router_bias=rb, w_gate=w_gate, w_up=w_up,
               w_down=w_down, sh_gate=sg, sh_up=su, sh_down=sd)
    if wl.weight_dtype == "fp8":
        # codes replace the fp32 draws; scales s_<name> [E, N] / [N]
        for name in ("w_gate", "w_up", "w_down", "sh_gate", "sh_up", "sh_down"):
            out[name], out["s_" + name] = quantize_e4m3(out[name])
    return out


def make_shard_inputs(wl: Workload, first: int, count: int, with_shared: bool,
                      device="cpu") -> Dict[str, torch.Tensor]:
    """The tensors an expert shard loads (moe_load_shard_weights): x, the
    whole router, experts [first, first + count) only ([count, ...]), and the
    shared expert if the shard holds it.  Each expert comes from its own
    generator, so these equal the matching slices of make_inputs."""
    dev = torch.device(device)
    x = draw_x(wl, dev)
    rw, rb = draw_router(wl, dev)
    H, I = wl.hidden, wl.intermediate
    dt = _torch_dtype(wl.weight_dtype)
    w_gate = torch.empty(count, H, I, dtype=dt, device=dev)
    w_up = torch.empty(count, H, I, dtype=dt, device=dev)
    w_down = torch.empty(count, I, H, dtype=dt, device=dev)
    for i in range(count):
        wg, wu, wd = draw_expert(wl, first + i, dev)
        w_gate[i].copy_(wg)
        w_up[i].copy_(wu)
        w_down[i].copy_(wd)
    out = dict(x=x, router_w=rw, router_bias=rb, w_gate=w_gate, w_up=w_up, w_down=w_down)
    if with_shared:
        out["sh_gate"], out["sh_up"], out["sh_down"] = draw_shared(wl, dev)
    return out


class HostExpertView:
    """``view[e]`` -> exact float32 host copy of expert e's matrix of a device
    tensor [E, ...]; lets the oracle walk a 9 GB weight set expert by expert."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __getitem__(self, e: int):
        return self.t[e].float().cpu().numpy()

    def __len__(self):
        return self.t.shape[0]


def host_f32(t: torch.Tensor):
    """Exact float32 host copy (bf16 widens exactly)."""
    return t.detach().float().cpu().numpy()


# ---------------------------------------------------------------- dense MLP

@dataclass(frozen=True)
class DenseWorkload:
    """The dense SwiGLU MLP of the first three decoder layers (no routing):
    x [T, H] -> out [T, H] through w_gate, w_up [H, I] and w_down [I, H]."""
    name: str
    T: int
    hidden: int
    intermediate: int
    act_dtype: str                 # "f32" or "bf16"
    weight_dtype: str              # "f32" or "bf16"
    x_dist: str                    # "normal" or "rmsnorm_normal"
    weight_std: float
    swiglu_limit: float = 0.0
    seed: int = 0
    description: str = ""

    def with_T(self, T: int) -> "DenseWorkload":
        return replace(self, T=T)


# stream ids of the dense MLP's tensors (disjoint from the MoE layer's)
_S_DENSE = 500

DENSE_WORKLOADS: Dict[str, DenseWorkload] = {
    "dense_tiny": DenseWorkload(
        name="dense_tiny", T=96, hidden=256, intermediate=320, act_dtype="f32",
        weight_dtype="f32", x_dist="normal", weight_std=0.05,
        description="T=96, H=256, I=320 (padded to 384), fp32"),
    "dense_decode": DenseWorkload(
        name="dense_decode", T=64, hidden=4096, intermediate=11264, act_dtype="bf16",
        weight_dtype="bf16", x_dist="rmsnorm_normal", weight_std=0.02,
        description="Step-3.5-Flash dense MLP layer (intermediate 11264), T=64"),
    "dense_prefill": DenseWorkload(
        name="dense_prefill", T=4096, hidden=4096, intermediate=11264, act_dtype="bf16",
        weight_dtype="bf16", x_dist="rmsnorm_normal", weight_std=0.02,
        description="Step-3.5-Flash dense MLP layer (intermediate 11264), T=4096"),
}


def make_dense_inputs(wl: DenseWorkload, device="cpu") -> Dict[str, torch.Tensor]:
    """x [T, H] (act dtype); w_gate, w_up [H, I]; w_down [I, H] (weight dtype)."""
    dev = torch.device(device)
    x = torch.randn(wl.T, wl.hidden, generator=_gen(dev, wl.seed, _S_DENSE),
                    device=dev, dtype=torch.float32)
    if wl.x_dist == "rmsnorm_normal":
        x = x / torch.sqrt(torch.mean(x * x, dim=1, keepdim=True))
    g = _gen(dev, wl.seed, _S_DENSE + 1)
    H, I = wl.hidden, wl.intermediate
    dt = _torch_dtype(wl.weight_dtype)
    wg = (torch.randn(H, I, generator=g, device=dev) * wl.weight_std).to(dt)
    wu = (torch.randn(H, I, generator=g, device=dev) * wl.weight_std).to(dt)
    wd = (torch.randn(I, H, generator=g, device=dev) * wl.weight_std).to(dt)
    return dict(x=x.to(_torch_dtype(wl.act_dtype)), w_gate=wg, w_up=wu, w_down=wd)
