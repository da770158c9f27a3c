"""CUDA-graph capture of the forwards.

A serving loop captures a forward once and replays it on whatever the
captured input buffer holds.  That works only if a forward enqueues nothing
but stream work -- no host synchronisation, no allocation, no host-side state
that a replay would not update (the dense stream-K launch therefore derives
its counter targets on the device).  Each case runs the forward eagerly on
two inputs, captures it, replays it twice on each input and asserts the
replays equal the eager outputs bit for bit.
"""
from dataclasses import replace

import pytest
import torch

from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import (DENSE_WORKLOADS, WORKLOADS, draw_x,
                                                  make_dense_inputs, make_inputs)

pytestmark = pytest.mark.gpu


def _check_replays(forward, x_static, out_static, xs):
    eager = []
    for x in xs:
        x_static.copy_(x)
        forward()
        torch.cuda.synchronize()
        eager.append(out_static.clone())
    # warm-up on a side stream, then capture (torch's recipe for graphs)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        forward()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        forward()
    for _ in range(2):
        for x, want in zip(xs, eager):
            x_static.copy_(x)
            out_static.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out_static, want)
    del g


MOE_CASES = {
    # one-SM tiles, CUDA-core router, block top-k, one-block sort
    "decode_like": (replace(WORKLOADS["tiny"], name="gd", T=64, hidden=512, num_experts=32,
                            top_k=4, intermediate=320, shared_intermediate=320,
                            act_dtype="bf16", weight_dtype="bf16", x_dist="rmsnorm_normal"),
                    "auto"),
    # CTA pairs, tensor-core router, warp top-k, three-kernel sort, row gather
    "pairs": (replace(WORKLOADS["tiny"], name="gp", T=2304, hidden=512, num_experts=24,
                      top_k=4, intermediate=256, shared_intermediate=256, act_dtype="bf16",
                      weight_dtype="bf16", x_dist="rmsnorm_normal"), "auto"),
    # the fused persistent forward (its counters are cleared inside the forward)
    "fused": (replace(WORKLOADS["tiny"], name="gf", T=2048, hidden=512, num_experts=32,
                      top_k=4, intermediate=256, shared_intermediate=256, act_dtype="bf16",
                      weight_dtype="bf16", x_dist="rmsnorm_normal"), "fused"),
    # the fp32 expert path
    "fp32": (WORKLOADS["tiny"], "auto"),
}


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name", list(MOE_CASES))
def test_moe_forward_graph_replay(name):
    wl, path = MOE_CASES[name]
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.set_path({"auto": B.MOE_PATH_AUTO, "fused": B.MOE_PATH_FUSED}[path])
    layer.load_inputs(inp)
    if path == "fused":
        assert B.moe_forward_path(layer.handle, wl.T) == B.MOE_PATH_FUSED
    xs = [inp["x"], draw_x(replace(wl, seed=7), "cpu").cuda()]
    x_static = torch.empty_like(xs[0])
    out_static = torch.empty_like(xs[0])
    _check_replays(lambda: layer.forward(x_static, out_static), x_static, out_static, xs)
    assert layer.device_error() == 0
    layer.close()


DENSE_CASES = {
    # up to 128 tokens with H % 256 == 0: the one-launch stream-K forward
    "streamk": replace(DENSE_WORKLOADS["dense_tiny"], name="gs", T=64, hidden=512,
                       intermediate=700, act_dtype="bf16", weight_dtype="bf16",
                       x_dist="rmsnorm_normal", swiglu_limit=0.8),
    # split-K GEMMs and their reduction kernels
    "splitk": replace(DENSE_WORKLOADS["dense_tiny"], name="gk", T=40, hidden=384,
                      intermediate=256, act_dtype="bf16", weight_dtype="bf16"),
    # the fp32 path
    "fp32": DENSE_WORKLOADS["dense_tiny"],
}


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name", list(DENSE_CASES))
def test_dense_forward_graph_replay(name):
    wl = DENSE_CASES[name]
    inp = {k: v.cuda() for k, v in make_dense_inputs(wl, "cpu").items()}
    layer = B.DenseMLP.from_workload(wl)
    layer.load_inputs(inp)
    x2 = make_dense_inputs(replace(wl, seed=7), "cpu")["x"].cuda()
    xs = [inp["x"], x2]
    x_static = torch.empty_like(xs[0])
    out_static = torch.empty_like(xs[0])
    _check_replays(lambda: layer.forward(x_static, out_static), x_static, out_static, xs)
    assert layer.device_error() == 0
    layer.close()
