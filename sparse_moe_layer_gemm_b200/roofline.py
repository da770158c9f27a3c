"""Roofline accounting of the MoE FFN layer forward: the bytes it must move at
least once and the flops it must execute, per workload and routing outcome."""
from __future__ import annotations

from .workloads import Workload


def _el_w(wl: Workload) -> int:
    """Bytes per expert weight: 1 for FP8 E4M3 codes, 2 bf16, 4 fp32."""
    return {"fp8": 1, "bf16": 2, "f32": 4}[wl.weight_dtype]


def _scale_bytes(wl: Workload, feats: int) -> int:
    """FP8 weights: one fp32 scale per output feature."""
    return 4 * feats if wl.weight_dtype == "fp8" else 0


def algorithmic_bytes(wl: Workload, touched_routed: int) -> int:
    """Bytes the layer must move at least once: the touched routed experts plus
    the shared expert (gate, up, down), the fp32 router weight and bias, the
    input x and the output (same dtype as x); FP8 weights add their scales."""
    el_w = _el_w(wl)
    el_x = 2 if wl.act_dtype == "bf16" else 4
    H, I, Is, E = wl.hidden, wl.intermediate, wl.shared_intermediate, wl.num_experts
    experts = touched_routed * (3 * H * I * el_w + _scale_bytes(wl, 2 * I + H)) + \
        3 * H * Is * el_w + _scale_bytes(wl, 2 * Is + H)
    router = H * E * 4 + E * 4
    act = 2 * wl.T * H * el_x
    return experts + router + act


def algorithmic_flops(wl: Workload) -> int:
    """Multiply-adds x2 of the router and of k routed + 1 shared SwiGLU experts."""
    H, I, Is, E, k = wl.hidden, wl.intermediate, wl.shared_intermediate, wl.num_experts, wl.top_k
    per_tok = 2 * H * E + k * (2 * H * 2 * I + 2 * I * H) + (2 * H * 2 * Is + 2 * Is * H)
    return wl.T * per_tok


def gate_up_bytes(wl: Workload, touched_routed: int) -> int:
    """Bytes the grouped gate|up GEMM must move at least once: the gate and up
    weights of the touched routed experts and of the shared expert, the input
    rows (T x H) and the SwiGLU output h ((k + 1) rows per token x I, bf16);
    FP8 weights add their scales."""
    el_w = _el_w(wl)
    el_x = 2 if wl.act_dtype == "bf16" else 4
    H, I = wl.hidden, wl.intermediate
    weights = (touched_routed + 1) * (2 * H * I * el_w + _scale_bytes(wl, 2 * I))
    return weights + wl.T * H * el_x + wl.T * (wl.top_k + 1) * I * 2


def gate_up_flops(wl: Workload) -> int:
    """2 x multiply-adds of the gate and up projections of k routed + 1 shared experts."""
    return wl.T * (wl.top_k + 1) * 2 * wl.hidden * 2 * wl.intermediate


def down_bytes(wl: Workload, touched_routed: int) -> int:
    """Down weights of the touched experts + shared (FP8: and their scales),
    h in, y out (bf16)."""
    H, I = wl.hidden, wl.intermediate
    rows = wl.T * (wl.top_k + 1)
    return (touched_routed + 1) * (H * I * _el_w(wl) + _scale_bytes(wl, H)) + \
        rows * I * 2 + rows * H * 2


def down_flops(wl: Workload) -> int:
    return wl.T * (wl.top_k + 1) * 2 * wl.intermediate * wl.hidden
