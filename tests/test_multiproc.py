"""The N > 1 host path on CPU with gloo, world size 2: replicas draw the same
weights and different batches, and the step time is the max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_moe_layer_gemm_b200.replicas import (job_throughput, max_over_ranks,
                                                 rank_batch_workload)
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, draw_expert, draw_x


def _free_port():
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
    mine = rank_batch_workload(wl, rank)
    x = draw_x(mine, "cpu")
    w = draw_expert(wl, 3, "cpu")[0]           # weights: the layer's own seed
    ms = 1.0 + rank                            # rank 1 is the slow one
    m = max_over_ranks(ms)
    xs = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(xs, x)
    ws = [torch.empty_like(w) for _ in range(world)]
    dist.all_gather(ws, w)
    q.put((rank, m, job_throughput(wl.T, world, m), not torch.equal(xs[0], xs[1]),
           torch.equal(ws[0], ws[1])))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_rank_replicas_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, thr, batches_differ, weights_same in res:
        assert m == 2.0                        # max over ranks
        assert thr == pytest.approx(2 * 32 / 2e-3)
        assert batches_differ and weights_same


def test_single_process_fallbacks():
    assert max_over_ranks(3.5) == 3.5
    assert job_throughput(64, 1, 1.0) == 64000.0
