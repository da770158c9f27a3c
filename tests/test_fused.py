"""The fused persistent forward (MOE_PATH_FUSED: router, top-k, counting sort,
both expert GEMMs and the combine in one launch, the pages' FusedEPMoE
backend) against the multi-launch path, bit for bit, and against the CPU
oracle, element by element.  The cases span narrow and wide token tiles, a
ragged last token block of the shared expert (narrow), distinct clamps, the
gathered token rows of many small experts and exact selection ties."""
from dataclasses import replace

import pytest
import torch

from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, host_f32, make_inputs
from tests.parity import compare, expert_views

pytestmark = pytest.mark.gpu

_BASE = dict(act_dtype="bf16", weight_dtype="bf16", x_dist="rmsnorm_normal")

FUSED = {
    # most experts hold a few rows: narrow tiles, gathered rows, 96 groups
    "narrow_tiles": replace(WORKLOADS["tiny"], name="fn", T=2048, hidden=512, num_experts=96,
                            top_k=4, intermediate=384, shared_intermediate=384,
                            swiglu_limit=0.9, swiglu_limit_shared=1.2, expert_std=0.08, **_BASE),
    # ~525 rows per expert: wide tiles, several token blocks per group
    "wide_tiles": replace(WORKLOADS["tiny"], name="fw", T=2100, hidden=512, num_experts=16,
                          top_k=4, intermediate=256, shared_intermediate=256,
                          swiglu_limit=0.9, swiglu_limit_shared=1.3, expert_std=0.08, **_BASE),
    # the shared expert's last token block has 40 rows (a narrow tile); 288
    # experts top-8 on a narrow hidden size; router rows past E_pad read 0
    "ragged_288": replace(WORKLOADS["tiny"], name="fr", T=2088, hidden=256, num_experts=288,
                          top_k=8, intermediate=128, shared_intermediate=128, **_BASE),
}


def _both_paths(wl, cpu):
    inp = {k: v.cuda() for k, v in cpu.items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    x = inp["x"]
    layer.set_path(B.MOE_PATH_MULTI)
    assert layer.forward_path(wl.T) == B.MOE_PATH_MULTI
    out_m, rt_m = layer.forward(x, routing=True)
    out_m = out_m.clone()
    rt_m = {k: v.clone() for k, v in rt_m.items()}
    layer.set_path(B.MOE_PATH_FUSED)
    assert layer.forward_path(wl.T) == B.MOE_PATH_FUSED
    assert B.moe_kernel_launches(layer.handle, wl.T) == 1
    out_f, rt_f = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    return layer, inp, out_m, rt_m, out_f, rt_f


def _check_same(out_m, rt_m, out_f, rt_f):
    for name in ("topk_idx", "topk_w", "counts", "offsets", "perm"):
        assert torch.equal(rt_f[name], rt_m[name]), name
    assert torch.equal(out_f, out_m), "fused and multi-launch outputs differ"


@pytest.mark.timeout(600)
@pytest.mark.parametrize("name", list(FUSED))
def test_fused_matches_multi_launch_and_oracle(name):
    wl = FUSED[name]
    cpu = make_inputs(wl, "cpu")
    layer, inp, out_m, rt_m, out_f, rt_f = _both_paths(wl, cpu)
    _check_same(out_m, rt_m, out_f, rt_f)
    host = {k: host_f32(cpu[k]) for k in ("x", "router_w", "router_bias")}
    rep = compare(host, wl, host_f32(out_f), {k: v.cpu().numpy() for k, v in rt_f.items()},
                  experts=expert_views(cpu))
    print(name, rep)
    assert rep.ok(), rep
    # a second fused forward gives the same bits (the counters start from zero)
    again = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert torch.equal(again, out_f)
    assert layer.device_error() == 0
    layer.close()


@pytest.mark.timeout(600)
def test_fused_exact_ties():
    """Duplicated router columns with equal biases: the tie rule (lower index
    first) decides, with no near-tie exception, on the fused path too."""
    wl = replace(FUSED["narrow_tiles"], name="ft", top_k=5)
    cpu = make_inputs(wl, "cpu")
    rw, rb = cpu["router_w"].clone(), cpu["router_bias"].clone()
    rw[:, 1::2] = rw[:, 0::2]
    rb[1::2] = rb[0::2]
    cpu["router_w"], cpu["router_bias"] = rw, rb
    layer, inp, out_m, rt_m, out_f, rt_f = _both_paths(wl, cpu)
    _check_same(out_m, rt_m, out_f, rt_f)
    host = {k: host_f32(cpu[k]) for k in ("x", "router_w", "router_bias")}
    rep = compare(host, wl, host_f32(out_f), {k: v.cpu().numpy() for k, v in rt_f.items()},
                  experts=expert_views(cpu), strict=True)
    assert rep.ok(), rep
    layer.close()


@pytest.mark.timeout(300)
def test_fused_not_eligible_falls_back():
    """fp32 x, fewer than 2048 tokens, or an expert shard: the multi-launch path."""
    wl = replace(FUSED["narrow_tiles"], act_dtype="f32")
    layer = B.MoeLayer.from_workload(wl)
    layer.set_path(B.MOE_PATH_FUSED)
    assert layer.forward_path(wl.T) == B.MOE_PATH_MULTI
    layer.close()
    wl = FUSED["narrow_tiles"]
    layer = B.MoeLayer.from_workload(wl)
    layer.set_path(B.MOE_PATH_FUSED)
    assert layer.forward_path(2047) == B.MOE_PATH_MULTI
    assert layer.forward_path(2048) == B.MOE_PATH_FUSED
    with pytest.raises(B.MoeError):
        layer.set_path(7)
    layer.close()
    shard = B.MoeLayer.from_workload(wl, shard=(0, 48, 1))
    shard.set_path(B.MOE_PATH_FUSED)
    assert shard.forward_path(wl.T) == B.MOE_PATH_MULTI
    shard.close()


@pytest.mark.timeout(300)
def test_fused_wait_runs_out_and_context_survives():
    """Fault detection without a fault, on the fused kernel itself: a forward
    in which no down tile can become ready (its readiness counter never
    reaches the target) with every wait limited to 20 ms.  The waits give up,
    every role winds down and frees its tensor memory, the status word holds
    exactly the timeout bit, and a normal fused forward afterwards still
    matches the multi-launch path bit for bit."""
    wl = FUSED["narrow_tiles"]
    cpu = make_inputs(wl, "cpu")
    inp = {k: v.cuda() for k, v in cpu.items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    layer.set_path(B.MOE_PATH_FUSED)
    x = inp["x"]
    out = torch.empty_like(x)
    ws = layer.workspace(wl.T)
    r, word = B.moe_check_fused_timeout(layer.handle, x, wl.T, out, ws, ws.numel(), 20000)
    assert r == B.MOE_OK, (B.status_string(r), word)
    assert word == 1
    fused = layer.forward(x).clone()
    layer.set_path(B.MOE_PATH_MULTI)
    multi = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert torch.equal(fused, multi)
    layer.close()
