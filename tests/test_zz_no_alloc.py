"""moe_route_static: routing with no device allocation.

Callers that cannot call cudaMalloc (code under CUDA-graph capture, runtimes
that own all device memory through their own pool, latency-critical loops
where an allocation could synchronise the device) route tokens through this
entry point; its scratch is a static device array inside the library.  This
test checks, through the C ABI, that two calls in a row give the same top-k
indices and gate weights as the routing outputs of moe_forward, so the
array's leftover contents from the first call do not leak into the second.
It runs the same alone in a fresh process or after the other tests.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, draw_x, make_inputs
from tests.parity import W_RTOL

pytestmark = pytest.mark.gpu


@pytest.mark.timeout(300)
def test_route_static_matches_forward_twice():
    # below 512 tokens moe_forward routes with the same CUDA-core kernels, so
    # the two entry points must agree bit for bit
    wl = replace(WORKLOADS["tiny"], name="noalloc", T=333, hidden=512, num_experts=32,
                 top_k=4, intermediate=320, shared_intermediate=320, act_dtype="bf16",
                 weight_dtype="bf16", x_dist="rmsnorm_normal")
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    batches = [inp["x"], draw_x(replace(wl, seed=11), "cpu").cuda()]
    for x in batches:                     # two calls in a row share the scratch array
        _, rt = layer.forward(x, routing=True)
        idx = torch.full((wl.T, wl.top_k), -1, dtype=torch.int32, device="cuda")
        w = torch.full((wl.T, wl.top_k), -1.0, dtype=torch.float32, device="cuda")
        r = B.moe_route_static(x, B.MOE_BF16, inp["router_w"], inp["router_bias"], wl.T,
                               wl.hidden, wl.num_experts, wl.top_k, True, wl.scale, idx, w)
        assert r == B.MOE_OK, B.status_string(r)
        torch.cuda.synchronize()
        assert torch.equal(idx, rt["topk_idx"])
        np.testing.assert_allclose(w.cpu().numpy(), rt["topk_w"].cpu().numpy(),
                                   rtol=W_RTOL, atol=1e-7)
    assert layer.device_error() == 0
    layer.close()


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
