"""moe_route_static: routing with no device allocation.

Callers that cannot call cudaMalloc (code under CUDA-graph capture, runtimes
that own all device memory through their own pool, latency-critical loops
where an allocation could synchronise the device) route tokens through this
entry point; its scratch is a static device array inside the library.  These
tests call it through the C ABI twice in a row on different batches (the
array keeps the first call's contents) and check each result against the CPU
oracle, and, where moe_forward routes with the same kernels, against
moe_forward's routing bit for bit.  They run the same alone in a fresh
process or after the other tests.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle.moe_oracle as om
from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import (WORKLOADS, draw_router, draw_x, host_f32,
                                                  make_inputs)
from tests.parity import W_RTOL, check_selection

pytestmark = pytest.mark.gpu


def _route_static(x, wl, rw, rb):
    idx = torch.full((wl.T, wl.top_k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((wl.T, wl.top_k), -1.0, dtype=torch.float32, device="cuda")
    dt = B.MOE_BF16 if x.dtype == torch.bfloat16 else B.MOE_F32
    r = B.moe_route_static(x, dt, rw, rb, wl.T, wl.hidden, wl.num_experts, wl.top_k, True,
                           wl.scale, idx, w)
    assert r == B.MOE_OK, B.status_string(r)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _check_oracle(x, wl, rw, rb, idx, w):
    ref = om.moe_routing(host_f32(x), host_f32(rw), host_f32(rb), top_k=wl.top_k,
                         scale=wl.scale)
    mism, tie = check_selection(idx, w, ref, wl.top_k, wl.num_experts, scale=wl.scale)
    return int(mism.sum()), int(tie.sum())


@pytest.mark.timeout(300)
def test_route_static_matches_forward_twice():
    # below 512 tokens moe_forward routes with the same CUDA-core kernels, so
    # the two entry points must agree bit for bit, and both with the oracle
    wl = replace(WORKLOADS["tiny"], name="noalloc", T=333, hidden=512, num_experts=32,
                 top_k=4, intermediate=320, shared_intermediate=320, act_dtype="bf16",
                 weight_dtype="bf16", x_dist="rmsnorm_normal")
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    batches = [inp["x"], draw_x(replace(wl, seed=11), "cpu").cuda()]
    for x in batches:                     # two calls in a row share the scratch array
        _, rt = layer.forward(x, routing=True)
        idx, w = _route_static(x, wl, inp["router_w"], inp["router_bias"])
        assert np.array_equal(idx, rt["topk_idx"].cpu().numpy())
        np.testing.assert_allclose(w, rt["topk_w"].cpu().numpy(), rtol=W_RTOL, atol=1e-7)
        _check_oracle(x, wl, inp["router_w"], inp["router_bias"], idx, w)
    assert layer.device_error() == 0
    layer.close()


# Regimes of its own, checked against the oracle (moe_forward routes these
# sizes with other kernels or another K split):
#   * T * E * H / 128 > 1,048,576: fewer K splits than moe_forward uses
#     (here 16 instead of 32), the usual case at the full layer's size;
#   * T >= 2048: the warp-per-token top-k (T * E <= 1,048,576 needs E <= 512;
#     the case below has more tokens than the full layer's prefill).
REGIMES = {
    "fewer_splits": replace(WORKLOADS["prefill"], name="ns", T=1024, num_experts=64),
    "warp_topk": replace(WORKLOADS["prefill"], name="wt", T=8448, hidden=256,
                         num_experts=96),
}


@pytest.mark.timeout(300)
@pytest.mark.parametrize("name", list(REGIMES))
def test_route_static_regimes_against_oracle(name):
    wl = REGIMES[name]
    rw, rb = draw_router(wl, "cpu")
    rw, rb = rw.cuda(), rb.cuda()
    for seed in (0, 5):                   # two calls in a row
        x = draw_x(replace(wl, seed=seed), "cpu").cuda()
        idx, w = _route_static(x, wl, rw, rb)
        mism, ties = _check_oracle(x, wl, rw, rb, idx, w)
        print(name, seed, "near-tied tokens", ties, "of them differing", mism)


@pytest.mark.timeout(60)
def test_route_static_rejects_oversize_without_launching():
    T, H, E, k = 4096, 512, 288, 8          # T * E > 1,048,576 partial logits
    x = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    rw = torch.zeros(H, E, dtype=torch.float32, device="cuda")
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    r = B.moe_route_static(x, B.MOE_BF16, rw, None, T, H, E, k, True, 3.0, idx, w)
    assert r == B.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((idx == -7).all()) and bool((w == -7.0).all())
