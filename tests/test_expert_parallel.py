"""Expert parallelism.  CPU (gloo, world size 2): the shard split covers
every expert once and the summed partial outputs equal the whole layer, with
the oracle standing in for each rank's kernels.  GPU (one device): shard
layers run one after another on the same GPU, and their partial outputs sum
to the oracle's output; the shard's routing counts are its own experts'."""
import os
import socket
from dataclasses import replace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.moe_oracle as om
from sparse_moe_layer_gemm_b200.expert_parallel import (holds_shared, reduce_partials,
                                                        shard_range)
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, host_f32, make_inputs


@pytest.mark.parametrize("E,world", [(288, 8), (288, 7), (16, 2), (5, 5), (13, 4)])
def test_shard_ranges_cover_once(E, world):
    seen = []
    for r in range(world):
        f, c = shard_range(E, world, r)
        assert c >= 1 and abs(c - E // world) <= 1
        seen.extend(range(f, f + c))
    assert seen == list(range(E))
    assert sum(holds_shared(r) for r in range(world)) == 1


def test_shard_range_rejects_bad_splits():
    with pytest.raises(ValueError):
        shard_range(3, 4, 0)
    with pytest.raises(ValueError):
        shard_range(16, 2, 2)


def _partial_oracle(inp, wl, first, count, with_shared):
    """The oracle's layer output restricted to one shard: the other experts'
    weights (and the shared expert's, if not held) set to zero, so their
    SwiGLU terms vanish while the routing (which does not read them) is the
    whole layer's."""
    keep = np.zeros(wl.num_experts, bool)
    keep[first:first + count] = True
    z = lambda a: np.where(keep[:, None, None], a, 0.0)
    sh = 1.0 if with_shared else 0.0
    return om.moe_forward(inp["x"], inp["router_w"], inp["router_bias"], z(inp["w_gate"]),
                          z(inp["w_up"]), z(inp["w_down"]), sh * inp["sh_gate"],
                          sh * inp["sh_up"], sh * inp["sh_down"], top_k=wl.top_k,
                          scale=wl.scale).out


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    wl = WORKLOADS["tiny"]
    inp = {k: host_f32(v).astype(np.float64) for k, v in make_inputs(wl, "cpu").items()}
    first, count = shard_range(wl.num_experts, world, rank)
    part = torch.from_numpy(_partial_oracle(inp, wl, first, count, holds_shared(rank)))
    total = reduce_partials(part.clone())
    full = om.moe_forward(inp["x"], inp["router_w"], inp["router_bias"], inp["w_gate"],
                          inp["w_up"], inp["w_down"], inp["sh_gate"], inp["sh_up"],
                          inp["sh_down"], top_k=wl.top_k, scale=wl.scale).out
    q.put((rank, float(np.max(np.abs(total.numpy() - full))), float(np.max(np.abs(full))),
           float(np.max(np.abs(part.numpy() - full)))))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_rank_partials_sum_to_layer_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale, part_err in res:
        assert err <= 1e-12 * scale          # fp64 sums of two partials
        assert part_err > 1e-3 * scale       # a partial alone is not the layer


@pytest.mark.gpu
@pytest.mark.timeout(300)
@pytest.mark.parametrize("case", ["two_shards", "three_uneven_fp32_x", "prefill_shape",
                                  "fp8_two_shards"])
def test_gpu_shards_sum_to_oracle(case):
    from sparse_moe_layer_gemm_b200 import binding as B
    from tests.parity import MAX_ABS_OVER_RMS, REL_FRO, output_errors
    if case == "two_shards":
        wl = replace(WORKLOADS["tiny"], name="ep2", T=200, act_dtype="bf16", weight_dtype="bf16")
        splits = [(0, 8, True), (8, 8, False)]
    elif case == "three_uneven_fp32_x":
        wl = replace(WORKLOADS["tiny"], name="ep3", T=300, num_experts=13, top_k=3)
        splits = [(0, 4, False), (4, 5, True), (9, 4, False)]
    elif case == "fp8_two_shards":  # FP8 codes and scales sliced per shard
        wl = replace(WORKLOADS["tiny"], name="ep8", T=150, hidden=512, num_experts=12, top_k=3,
                     intermediate=256, shared_intermediate=256, act_dtype="bf16",
                     weight_dtype="fp8", x_dist="rmsnorm_normal")
        splits = [(0, 5, False), (5, 7, True)]
    else:  # bulk-copy gather (bf16, >= 1024 tokens) and CTA pairs (>= 2048)
        wl = replace(WORKLOADS["tiny"], name="epp", T=2100, hidden=512, num_experts=16, top_k=4,
                     intermediate=256, shared_intermediate=256, act_dtype="bf16",
                     weight_dtype="bf16", x_dist="rmsnorm_normal")
        splits = [(0, 6, False), (6, 10, True)]
    cpu = make_inputs(wl, "cpu")
    inp = {k: v.cuda() for k, v in cpu.items()}
    total = None
    for first, count, sh in splits:
        layer = B.MoeLayer.from_workload(wl, (first, count, sh))
        layer.load_inputs(inp)
        out, rt = layer.forward(inp["x"], routing=True)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        sel = rt["topk_idx"].cpu().numpy()
        want = np.bincount(sel.ravel(), minlength=wl.num_experts)[first:first + count]
        assert np.array_equal(rt["counts"].cpu().numpy()[:count], want)
        part = out.float().cpu()
        total = part if total is None else total + part
        layer.close()
    from tests.parity import expert_views
    host = {k: host_f32(cpu[k]) for k in ("x", "router_w", "router_bias")}
    ev = expert_views(cpu)
    ref = om.moe_forward(host["x"], host["router_w"], host["router_bias"], ev["w_gate"],
                         ev["w_up"], ev["w_down"], ev["sh_gate"], ev["sh_up"], ev["sh_down"],
                         top_k=wl.top_k, scale=wl.scale).out
    rel, mx, _ = output_errors(total.numpy(), ref)
    assert rel <= REL_FRO and mx <= MAX_ABS_OVER_RMS, (rel, mx)


def test_shard_inputs_are_slices_of_the_layer():
    """What a rank of the expert-parallel bench draws (its experts only)
    equals the matching slices of the whole layer's tensors."""
    from sparse_moe_layer_gemm_b200.workloads import make_shard_inputs
    wl = WORKLOADS["tiny"]
    full = make_inputs(wl, "cpu")
    for first, count, sh in ((0, 5, True), (5, 11, False)):
        part = make_shard_inputs(wl, first, count, sh, "cpu")
        for n in ("x", "router_w", "router_bias"):
            assert torch.equal(part[n], full[n])
        for n in ("w_gate", "w_up", "w_down"):
            assert torch.equal(part[n], full[n][first:first + count])
        assert ("sh_gate" in part) == sh
        if sh:
            for n in ("sh_gate", "sh_up", "sh_down"):
                assert torch.equal(part[n], full[n])


def test_bench_ep_plan_covers_experts_once():
    import bench
    for E, world in ((288, 8), (288, 2), (16, 3)):
        seen, shared = [], 0
        for r in range(world):
            pl = bench.ep_plan(E, world, r)
            seen.extend(range(pl["first"], pl["first"] + pl["count"]))
            shared += pl["with_shared"]
        assert seen == list(range(E)) and shared == 1
    cfg = bench.ep_config(WORKLOADS["decode"], 8)
    assert cfg["parallelism"].startswith("ep8") and cfg["workload"] == "decode"


def _ep_bench_worker(rank, world, port, q):
    """One rank of the bench's expert-parallel step on the CPU: its own
    shard's tensors only, its partial output (the oracle standing in for the
    kernels), then the all-reduce the bench runs after every forward."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    import bench
    from sparse_moe_layer_gemm_b200.workloads import make_shard_inputs
    wl = WORKLOADS["tiny"]
    pl = bench.ep_plan(wl.num_experts, world, rank)
    part_in = {k: host_f32(v).astype(np.float64)
               for k, v in make_shard_inputs(wl, pl["first"], pl["count"], pl["with_shared"],
                                             "cpu").items()}
    E, H, I = wl.num_experts, wl.hidden, wl.intermediate
    f, c = pl["first"], pl["count"]
    wg = np.zeros((E, H, I)); wu = np.zeros((E, H, I)); wd = np.zeros((E, I, H))
    wg[f:f + c], wu[f:f + c], wd[f:f + c] = part_in["w_gate"], part_in["w_up"], part_in["w_down"]
    zs = np.zeros((H, wl.shared_intermediate))
    sg = part_in.get("sh_gate", zs)
    su = part_in.get("sh_up", zs)
    sd = part_in.get("sh_down", zs.T)
    part = om.moe_forward(part_in["x"], part_in["router_w"], part_in["router_bias"], wg, wu, wd,
                          sg, su, sd, top_k=wl.top_k, scale=wl.scale).out
    total = reduce_partials(torch.from_numpy(part.copy()))
    full_in = {k: host_f32(v).astype(np.float64) for k, v in make_inputs(wl, "cpu").items()}
    full = om.moe_forward(full_in["x"], full_in["router_w"], full_in["router_bias"],
                          full_in["w_gate"], full_in["w_up"], full_in["w_down"],
                          full_in["sh_gate"], full_in["sh_up"], full_in["sh_down"],
                          top_k=wl.top_k, scale=wl.scale).out
    q.put((rank, float(np.max(np.abs(total.numpy() - full))), float(np.max(np.abs(full)))))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_bench_ep_step_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_ep_bench_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale in res:
        assert err <= 1e-12 * scale


@pytest.mark.gpu
@pytest.mark.timeout(300)
def test_gpu_shard_only_loading_matches_full_loading():
    """moe_load_shard_weights with a shard's own experts gives the same bits
    as moe_load_weights with the whole tensors."""
    from sparse_moe_layer_gemm_b200 import binding as B
    from sparse_moe_layer_gemm_b200.workloads import make_shard_inputs
    wl = replace(WORKLOADS["tiny"], name="eps", T=300, act_dtype="bf16", weight_dtype="bf16")
    full = {k: v.cuda() for k, v in make_inputs(wl, "cpu").items()}
    for first, count, sh in ((0, 7, True), (7, 9, False)):
        a = B.MoeLayer.from_workload(wl, (first, count, sh))
        a.load_inputs(full)
        b = B.MoeLayer.from_workload(wl, (first, count, sh))
        part = {k: v.cuda() for k, v in make_shard_inputs(wl, first, count, sh, "cpu").items()}
        b.load_shard_weights(part["router_w"], part["router_bias"], part["w_gate"], part["w_up"],
                             part["w_down"], part.get("sh_gate"), part.get("sh_up"),
                             part.get("sh_down"))
        oa = a.forward(full["x"]).clone()
        ob = b.forward(full["x"])
        torch.cuda.synchronize()
        assert a.device_error() == 0 and b.device_error() == 0
        assert torch.equal(oa, ob)
        a.close()
        b.close()
