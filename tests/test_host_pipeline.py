"""The pipelined host-buffer forward (moe_forward_host_async / _join): a
stream of batches with their own pinned input and output buffers, the
staging slots alternating, each result bit-identical to the device forward
of the same batch."""
import pytest
import torch

from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, make_inputs
from dataclasses import replace

pytestmark = pytest.mark.gpu


@pytest.mark.timeout(300)
@pytest.mark.parametrize("T", [200, 2100])  # one-SM tiles; CTA pairs
def test_pipelined_host_forward_matches_device_forward(T):
    wl = replace(WORKLOADS["tiny"], name="hp", T=T, hidden=512, num_experts=24, top_k=4,
                 intermediate=256, shared_intermediate=256, act_dtype="bf16",
                 weight_dtype="bf16", x_dist="rmsnorm_normal")
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    g = torch.Generator().manual_seed(3)
    xs = [(inp["x"].float().cpu() * (0.5 + i) + 0.01 * torch.randn(inp["x"].shape, generator=g))
          .to(torch.bfloat16).pin_memory() for i in range(5)]
    # two more batches of another T (the staging slots move)
    xs += [x[: T // 2 + 1].clone().pin_memory() for x in xs[:2]]
    outs = [torch.empty_like(x).pin_memory() for x in xs]
    stream = torch.cuda.Stream()
    layer.workspace(T, host_io=True)  # sized for the largest T up front
    for x, o in zip(xs, outs):
        layer.forward_host_async(x, o, stream=stream)
    layer.forward_host_join(stream=stream)
    stream.synchronize()
    for x, o in zip(xs, outs):
        ref = layer.forward(x.cuda())
        torch.cuda.synchronize()
        assert torch.equal(o, ref.cpu())
    assert layer.device_error() == 0
    layer.close()
