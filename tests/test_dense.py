"""GPU parity of the dense SwiGLU MLP (the first three decoder layers) with
the CPU oracle: small shapes compared on every row (several weight tiles,
padded I, ragged T, both tile schedules), the full-size decode and prefill
shapes on sampled rows.  Layers with fp32 weights take the fp32 path and
meet its tighter bar (tests/parity.py)."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle.moe_oracle as om
from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import DENSE_WORKLOADS, host_f32, make_dense_inputs
from tests.parity import (BF16_U, MAX_ABS_OVER_RMS, MAX_ABS_OVER_RMS_F32, REL_FRO, REL_FRO_F32,
                          fp32_bar_scale, output_errors)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny_fp32": DENSE_WORKLOADS["dense_tiny"],
    "bf16_clamped_ragged": replace(DENSE_WORKLOADS["dense_tiny"], name="dc", T=333, hidden=512,
                                   intermediate=700, act_dtype="bf16", weight_dtype="bf16",
                                   x_dist="rmsnorm_normal", swiglu_limit=0.8),
    "one_token": replace(DENSE_WORKLOADS["dense_tiny"], name="d1", T=1, act_dtype="bf16",
                         weight_dtype="bf16"),
    # from 2048 tokens: CTA pairs, 256-token tiles, and a ragged last tile
    "pairs_ragged": replace(DENSE_WORKLOADS["dense_tiny"], name="dp", T=2100, hidden=512,
                            intermediate=384, act_dtype="bf16", weight_dtype="bf16",
                            x_dist="rmsnorm_normal"),
    # odd H / 128: down tiles of one 128-feature block (fp32 path; bf16
    # weights with fp32 x)
    "odd_hidden_fp32": replace(DENSE_WORKLOADS["dense_tiny"], name="do", T=150, hidden=384,
                               intermediate=256),
    "odd_hidden_bf16_w": replace(DENSE_WORKLOADS["dense_tiny"], name="dw", T=150, hidden=384,
                                 intermediate=256, weight_dtype="bf16"),
    # the fp32 path at sizes the bf16 weights would run on CTA pairs, and
    # with bf16 x (bf16 output: its own rounding set apart)
    "fp32_many_tokens": replace(DENSE_WORKLOADS["dense_tiny"], name="dm", T=2100, hidden=512,
                                intermediate=384),
    "fp32_w_bf16_x": replace(DENSE_WORKLOADS["dense_tiny"], name="dx", T=77, hidden=512,
                             intermediate=700, act_dtype="bf16", x_dist="rmsnorm_normal",
                             swiglu_limit=0.8),
    # up to 128 tokens with H % 256 == 0: the one-launch stream-K forward.
    # Ragged T (not a multiple of 16), padded I, fewer (tile, K block) units
    # than SMs in both GEMMs (CTAs with empty ranges), clamped SwiGLU:
    "streamk_ragged_clamped": replace(DENSE_WORKLOADS["dense_tiny"], name="ds", T=77, hidden=512,
                                      intermediate=700, act_dtype="bf16", weight_dtype="bf16",
                                      x_dist="rmsnorm_normal", swiglu_limit=0.8),
    # more units than SMs in both GEMMs (every CTA holds one or two segments),
    # a full 128-token block, fp32 activations (bf16 weights)
    "streamk_full_block_fp32": replace(DENSE_WORKLOADS["dense_tiny"], name="df", T=128,
                                       hidden=1024, intermediate=2560, weight_dtype="bf16"),
    # H % 256 != 0 at decode-sized T: the split-K GEMMs and reduction kernels
    "splitk_odd_hidden": replace(DENSE_WORKLOADS["dense_tiny"], name="dk", T=40, hidden=384,
                                 intermediate=256, act_dtype="bf16", weight_dtype="bf16"),
}


def _run(wl, rows=None):
    cpu_or_dev = "cpu" if wl.hidden * wl.intermediate < (1 << 24) else "cuda"
    inp = {k: v.cuda() for k, v in make_dense_inputs(wl, cpu_or_dev).items()}
    layer = B.DenseMLP.from_workload(wl)
    layer.load_inputs(inp)
    out = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    rows = np.arange(wl.T) if rows is None else rows
    x = host_f32(inp["x"])[rows]
    ref = om.dense_mlp(x, host_f32(inp["w_gate"]), host_f32(inp["w_up"]),
                       host_f32(inp["w_down"]), wl.swiglu_limit)
    rel, mx, ex = output_errors(host_f32(out)[rows], ref)
    layer.close()
    return rel, mx, ex


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name", list(SMALL))
def test_dense_small_parity(name):
    wl = SMALL[name]
    rel, mx, ex = _run(wl)
    assert rel <= REL_FRO and mx <= MAX_ABS_OVER_RMS, (rel, mx)
    if wl.weight_dtype == "f32":  # the fp32 path's bar
        sc = fp32_bar_scale(wl.hidden, wl.intermediate)
        if wl.act_dtype == "bf16":
            assert rel <= BF16_U + REL_FRO_F32 * sc and \
                ex <= MAX_ABS_OVER_RMS_F32 * sc * (1 + BF16_U), (rel, ex)
        else:
            assert rel <= REL_FRO_F32 * sc and mx <= MAX_ABS_OVER_RMS_F32 * sc, (rel, mx)


@pytest.mark.timeout(600)
@pytest.mark.parametrize("name", ["dense_decode", "dense_prefill"])
def test_dense_full_size_parity(name):
    wl = DENSE_WORKLOADS[name]
    rng = np.random.default_rng(5)
    # decode: every row (seconds of oracle time); prefill: sampled rows
    rows = (np.arange(wl.T) if wl.T <= 128 else
            np.unique(np.concatenate([[0, wl.T - 1], rng.integers(0, wl.T, 24)])))
    rel, mx, _ = _run(wl, rows)
    assert rel <= REL_FRO and mx <= MAX_ABS_OVER_RMS, (rel, mx)


@pytest.mark.timeout(120)
def test_dense_deterministic_and_batch_independent():
    wl = SMALL["bf16_clamped_ragged"]
    inp = {k: v.cuda() for k, v in make_dense_inputs(wl, "cpu").items()}
    layer = B.DenseMLP.from_workload(wl)
    layer.load_inputs(inp)
    a = layer.forward(inp["x"]).clone()
    b = layer.forward(inp["x"]).clone()
    part = layer.forward(inp["x"][100:250].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(part, a[100:250])
    layer.close()


@pytest.mark.timeout(120)
def test_dense_streamk_deterministic_and_batch_independent():
    """The stream-K forward splits K by (tile, K block) units, which do not
    depend on T: the same rows give bit-identical outputs in any batch of up
    to 128 tokens, and twice in a row."""
    wl = SMALL["streamk_ragged_clamped"]
    inp = {k: v.cuda() for k, v in make_dense_inputs(wl, "cpu").items()}
    layer = B.DenseMLP.from_workload(wl)
    layer.load_inputs(inp)
    a = layer.forward(inp["x"]).clone()
    b = layer.forward(inp["x"]).clone()
    part = layer.forward(inp["x"][30:50].contiguous())
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    assert torch.equal(a, b)
    assert torch.equal(part, a[30:50])
    layer.close()
