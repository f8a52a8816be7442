"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks, the slowest
rank's time wins and the job's value counts every rank's copy of the
workload (weak scaling, no collective on the data path)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads as W
        ms = [1.25, 2.5][rank]
        slowest = bench.max_over_ranks(ms, world, torch.device("cpu"))
        w = W.WORKLOADS["sla2_bf16"]
        q.put((rank, slowest, bench.whole_job_value(w, world, slowest)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_weak_scaling_value():
    import workloads as W
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    w = W.WORKLOADS["sla2_bf16"]
    want = 2 * w.dense_equiv_flops() / 2.5e-3 / 1e12
    for rank, slowest, value in got:
        assert slowest == 2.5
        assert value == pytest.approx(want)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
