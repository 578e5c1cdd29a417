"""The bench's multi-rank aggregation (one process per GPU, replicas): the job
time is the slowest rank's device time and the job throughput is world x one
replica's work over it.  Run as two gloo ranks on the CPU."""
import os
import socket

import pytest
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
        total_ms = [10.0, 14.0][rank]  # rank 1 is the slower one
        q.put((rank, bench.aggregate(total_ms, steps=2, flops=1e12, tokens=1000, world=world, dist=dist,
                                     device="cpu")))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    for rank in (0, 1):
        ms, tflops, value, tokens_s = res[rank]
        assert ms == pytest.approx(7.0)              # max(10, 14) / 2 steps
        assert tflops == pytest.approx(1e12 / 7e-3 / 1e12)
        assert value == pytest.approx(2 * tflops)    # two replicas
        assert tokens_s == pytest.approx(2 * 1000 / 7e-3)
