"""Fault detection without a fault: a bounded wait that nothing satisfies
gives up, reports the timeout bit in the device status word, and the CUDA
context stays usable (a forward runs and matches the oracle afterwards)."""
import time

import pytest
import torch

from sparse_moe_layer_gemm_b200 import binding as B
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, host_f32, make_inputs
from tests.parity import compare

pytestmark = pytest.mark.gpu


@pytest.mark.timeout(120)
def test_wait_gives_up_and_reports():
    t0 = time.time()
    r, word = B.moe_check_wait_timeout(20000)  # 20 ms
    took = time.time() - t0
    assert r == B.MOE_OK, (r, word)
    assert word == 1                            # the timeout bit, nothing else
    assert took < 30.0
    # the context is still usable
    wl = WORKLOADS["tiny"]
    inp = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    layer = B.MoeLayer.from_workload(wl)
    layer.load_inputs(inp)
    out, rt = layer.forward(inp["x"], routing=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    rep = compare({k: host_f32(v) for k, v in inp.items()}, wl, host_f32(out),
                  {k: v.cpu().numpy() for k, v in rt.items()})
    layer.close()
    assert rep.ok(), rep

