"""GPU parity of the CUDA path (through the C ABI) with the CPU oracle.

Small shapes are compared on every row; they span several weight and token
tiles, padded intermediate sizes and ragged tails.  The five workloads run at
their full sizes in the launch configuration the benchmark times and are
compared on sampled rows (plus every near-tied row), with the routing checked
for every token.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import (WORKLOADS, HostExpertView, draw_router,
                                                  draw_x, host_f32, make_inputs)
from tests.parity import compare, expert_views

pytestmark = pytest.mark.gpu


def _routing_np(rt):
    return {k: v.cpu().numpy() for k, v in rt.items()}


def _run_small(wl):
    cpu = make_inputs(wl, "cpu")
    inp = {k: v.cuda() for k, v in cpu.items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    out, rt = layer.forward(inp["x"], routing=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    host = {k: host_f32(cpu[k]) for k in ("x", "router_w", "router_bias")}
    rep = compare(host, wl, host_f32(out), _routing_np(rt), experts=expert_views(cpu))
    layer.close()
    return rep


SMALL = {
    "tiny": WORKLOADS["tiny"],
    # 3 weight tiles of gate/up (I = 320 padded to 384), 4 of down, 8 K-blocks
    "multi_tile_ragged": replace(WORKLOADS["tiny"], name="mtr", T=777, hidden=512,
                                 num_experts=32, top_k=4, intermediate=320,
                                 shared_intermediate=320, act_dtype="bf16",
                                 weight_dtype="bf16", x_dist="rmsnorm_normal"),
    # ~375 rows per expert: three token tiles per group plus a ragged one
    "few_experts_many_rows": replace(WORKLOADS["tiny"], name="fe", T=1500, hidden=256,
                                     num_experts=8, top_k=2, intermediate=128,
                                     shared_intermediate=128, act_dtype="bf16",
                                     weight_dtype="bf16", bias="zero"),
    "clamped": replace(WORKLOADS["tiny"], name="cl", T=200, hidden=384, num_experts=24,
                       top_k=6, intermediate=192, shared_intermediate=192,
                       swiglu_limit=0.6, swiglu_limit_shared=0.8, expert_std=0.08),
    "fp32_x_bf16_w": replace(WORKLOADS["tiny"], name="xw", T=96, weight_dtype="bf16"),
    "single_token": replace(WORKLOADS["tiny"], name="t1", T=1, act_dtype="bf16",
                            weight_dtype="bf16"),
    "five_tokens": replace(WORKLOADS["tiny"], name="t5", T=5, act_dtype="bf16",
                           weight_dtype="bf16"),
    "top1_of_1": replace(WORKLOADS["tiny"], name="e1", T=64, num_experts=1, top_k=1),
    # many token tiles per group: ~525 rows per expert = four full token tiles
    # and a ragged one; down tiles of two weight blocks
    "large_tiles": replace(WORKLOADS["tiny"], name="lt", T=2100, hidden=512, num_experts=16,
                           top_k=4, intermediate=256, shared_intermediate=256,
                           act_dtype="bf16", weight_dtype="bf16", x_dist="rmsnorm_normal",
                           swiglu_limit=0.9, swiglu_limit_shared=1.3, expert_std=0.08),
    # H with an odd number of 128-feature blocks: down tiles of one block
    "large_odd_hidden": replace(WORKLOADS["tiny"], name="lo", T=2048, hidden=384,
                                num_experts=12, top_k=3, intermediate=128,
                                shared_intermediate=128, act_dtype="bf16", weight_dtype="bf16"),
    # fp32 x on CTA pairs: CUDA-core router, row gather with the shared rows
    # in x_perm, pair GEMMs reading them; some experts with a handful of rows
    "large_fp32_x": replace(WORKLOADS["tiny"], name="lf", T=2304, hidden=512, num_experts=24,
                            top_k=4, intermediate=256, shared_intermediate=256,
                            act_dtype="f32", weight_dtype="bf16", swiglu_limit=0.9,
                            swiglu_limit_shared=1.1, expert_std=0.08),
    # CTA pairs with mostly narrow tiles (a median of ~12 rows per expert,
    # 80 of 96 experts at most 128): MMAs of 16-144 columns next to the shared
    # expert's full 256-token tiles in one CTA's sequence; down with an odd
    # number of K stages (I = 384: three)
    "pair_narrow_tiles": replace(WORKLOADS["tiny"], name="pn", T=2048, hidden=512,
                                 num_experts=96, top_k=4, intermediate=384,
                                 shared_intermediate=384, act_dtype="bf16",
                                 weight_dtype="bf16", x_dist="rmsnorm_normal",
                                 swiglu_limit=0.9, swiglu_limit_shared=1.2, expert_std=0.08),
    # tensor-core router with the warp-per-token top-k (from 8192 tokens) on a
    # small layer
    "many_tokens_small_layer": replace(WORKLOADS["tiny"], name="mt", T=8448, hidden=256,
                                       num_experts=40, top_k=6, intermediate=128,
                                       shared_intermediate=128, act_dtype="bf16",
                                       weight_dtype="bf16", x_dist="rmsnorm_normal"),
    # FP8 E4M3 expert weights (codes + per-feature scales), one-SM tiles with
    # converter warps at every size: padded I (320 -> 384) with two-block down
    # tiles; odd H (one-block down tiles) with fp32 x; many rows per expert
    # with the clamp; one token
    "fp8_multi_tile_ragged": replace(WORKLOADS["tiny"], name="f8m", T=777, hidden=512,
                                     num_experts=32, top_k=4, intermediate=320,
                                     shared_intermediate=320, act_dtype="bf16",
                                     weight_dtype="fp8", x_dist="rmsnorm_normal"),
    "fp8_odd_hidden_fp32_x": replace(WORKLOADS["tiny"], name="f8o", T=300, hidden=384,
                                     num_experts=12, top_k=3, intermediate=128,
                                     shared_intermediate=128, weight_dtype="fp8"),
    "fp8_clamped_many_rows": replace(WORKLOADS["tiny"], name="f8c", T=2100, hidden=512,
                                     num_experts=16, top_k=4, intermediate=256,
                                     shared_intermediate=256, act_dtype="bf16",
                                     weight_dtype="fp8", x_dist="rmsnorm_normal",
                                     swiglu_limit=0.9, swiglu_limit_shared=1.3,
                                     expert_std=0.08),
    "fp8_single_token": replace(WORKLOADS["tiny"], name="f81", T=1, act_dtype="bf16",
                                weight_dtype="fp8"),
    # an odd number of pipeline stages per gate|up tile (H = 384: three) and
    # many tiles per CTA, so the issuers' stage parity alternates from tile
    # to tile
    "fp8_odd_stages_many_tiles": replace(WORKLOADS["tiny"], name="f8s", T=1500, hidden=384,
                                         num_experts=12, top_k=3, intermediate=192,
                                         shared_intermediate=192, act_dtype="bf16",
                                         weight_dtype="fp8", x_dist="rmsnorm_normal"),
}


@pytest.mark.timeout(120)
def test_fp8_decode_every_code():
    """The GEMMs' E4M3 -> bf16 converter on all 256 codes: every finite code
    gives the oracle's value exactly (bf16 holds them all), subnormals
    included; the two NaN codes give +-480 (the format excludes them)."""
    import oracle.moe_oracle as om
    codes = torch.arange(256, dtype=torch.uint8, device="cuda")
    got = B.moe_decode_e4m3(codes).float().cpu().numpy().astype(np.float64)
    want = om.decode_e4m3(np.arange(256))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    assert got[0x7F] == 480.0 and got[0xFF] == -480.0
    assert np.signbit(got[0x80])


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(name):
    rep = _run_small(SMALL[name])
    assert rep.ok(), rep


@pytest.mark.timeout(300)
def test_determinism_and_entry_points():
    wl = SMALL["multi_tile_ragged"]
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    a = layer.forward(inp["x"]).clone()
    b = layer.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b), "two forwards differ"
    # host-buffer entry point gives the same bits
    xh = inp["x"].cpu().pin_memory()
    oh = layer.forward_host(xh)
    assert torch.equal(oh, a.cpu())
    # one-shot entry point gives the same bits
    out = torch.empty_like(inp["x"])
    r = B.moe_forward_oneshot(inp["x"], inp["router_w"], inp["router_bias"], inp["w_gate"],
                              inp["w_up"], inp["w_down"], inp["sh_gate"], inp["sh_up"],
                              inp["sh_down"], wl.T, wl.hidden, wl.num_experts, wl.top_k,
                              wl.intermediate, wl.scale, wl.swiglu_limit,
                              wl.swiglu_limit_shared, B.MOE_BF16, B.MOE_BF16, out)
    assert r == B.MOE_OK
    torch.cuda.synchronize()
    assert torch.equal(out, a)
    # a row's output does not depend on the other rows of its batch: checked
    # within each router regime (tensor cores from 512 bf16 tokens, CUDA
    # cores below; across the two the router logits differ by fp32 rounding)
    part = layer.forward(inp["x"][100:700].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(part, a[100:700])
    small = layer.forward(inp["x"][:300].contiguous()).clone()
    smaller = layer.forward(inp["x"][40:97].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(smaller, small[40:97])
    assert layer.device_error() == 0
    layer.close()


@pytest.mark.timeout(120)
def test_host_checks_launch_nothing():
    wl = WORKLOADS["tiny"]
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    x = inp["x"]
    out = torch.full_like(x, 7.0)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    # weights not loaded yet
    assert B.moe_forward(layer.handle, x.data_ptr(), wl.T, out.data_ptr(), ws.data_ptr(),
                         ws.numel()) == B.MOE_ERR_NOT_LOADED
    layer.load_inputs(inp)
    need = B.moe_workspace_size(layer.handle, wl.T)
    assert B.moe_forward(layer.handle, x.data_ptr(), wl.T, out.data_ptr(), ws.data_ptr(),
                         need - 1) == B.MOE_ERR_WORKSPACE
    assert B.moe_forward(layer.handle, x.data_ptr(), wl.T, out.data_ptr(), ws.data_ptr() + 8,
                         ws.numel() - 8) == B.MOE_ERR_WORKSPACE
    assert B.moe_forward(layer.handle, x.data_ptr(), wl.T, x.data_ptr(), ws.data_ptr(),
                         ws.numel()) == B.MOE_ERR_INVALID_ARG
    assert B.moe_forward(layer.handle, x.data_ptr(), 0, out.data_ptr(), 0, 0) == B.MOE_OK
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "a rejected call wrote the output"
    assert B.moe_workspace_size(layer.handle, 0) == 0
    layer.close()


# ---------------------------------------------------------------- full sizes

@pytest.fixture(scope="module")
def step35():
    """The Step-3.5-Flash layer with N(0, 0.02) bf16 expert weights (shared
    by the decode, prefill and Zipf workloads), drawn on the device."""
    wl = WORKLOADS["decode"]
    inp = make_inputs(wl, "cuda")
    layer = B.MoeLayer.from_workload(wl)
    yield wl, inp, layer
    layer.close()
    del inp
    torch.cuda.empty_cache()


def _full(wl, inp, layer, n_rows=24):
    rw, rb = draw_router(wl, "cuda")
    layer.load_weights(inp["router_w"], rb, inp["w_gate"], inp["w_up"], inp["w_down"],
                       inp["sh_gate"], inp["sh_up"], inp["sh_down"])
    assert torch.equal(rw, inp["router_w"])
    x = draw_x(wl, "cuda")
    out, rt = layer.forward(x, routing=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    host = dict(x=host_f32(x), router_w=host_f32(inp["router_w"]), router_bias=host_f32(rb))
    experts = dict(w_gate=HostExpertView(inp["w_gate"]), w_up=HostExpertView(inp["w_up"]),
                   w_down=HostExpertView(inp["w_down"]), sh_gate=host_f32(inp["sh_gate"]),
                   sh_up=host_f32(inp["sh_up"]), sh_down=host_f32(inp["sh_down"]))
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, wl.T - 1], rng.integers(0, wl.T, n_rows)]))
    rep = compare(host, wl, host_f32(out), _routing_np(rt), rows=rows, experts=experts)
    print(wl.name, rep)
    return rep


@pytest.mark.timeout(900)
@pytest.mark.parametrize("name", ["decode", "prefill", "zipf_prefill"])
def test_full_size_parity(step35, name):
    _, inp, layer = step35
    rep = _full(WORKLOADS[name], inp, layer)
    assert rep.ok(), rep


@pytest.mark.timeout(900)
def test_full_size_clamp_ragged():
    wl = WORKLOADS["clamp_ragged"]
    inp = make_inputs(wl, "cuda")
    layer = B.MoeLayer.from_workload(wl)
    rep = _full(wl, inp, layer)
    layer.close()
    assert rep.ok(), rep


@pytest.mark.timeout(900)
def test_full_size_fp8_decode():
    """The decode workload with FP8 E4M3 expert weights (the fp32 draws
    quantised per output feature), at full size, sampled rows."""
    wl = replace(WORKLOADS["decode"], name="decode_fp8", weight_dtype="fp8")
    inp = make_inputs(wl, "cuda")
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    out, rt = layer.forward(inp["x"], routing=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    host = {k: host_f32(inp[k]) for k in ("x", "router_w", "router_bias")}
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([[0, wl.T - 1], rng.integers(0, wl.T, 24)]))
    rep = compare(host, wl, host_f32(out), _routing_np(rt), rows=rows,
                  experts=expert_views(inp))
    print(wl.name, rep)
    layer.close()
    assert rep.ok(), rep
