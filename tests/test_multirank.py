"""The multi-GPU host logic of bench.py on CPU: two gloo ranks, each with its
own replica and its own step time; both must agree on the slowest rank's time
and on the whole-job throughput.  No GPU needed."""
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
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    total = bench.max_over_ranks(local_ms, dist)
    ms, value = bench.throughput(total, steps=5, world=world, flops_per_step=1e12)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, total, ms, value))


def test_two_ranks_agree_on_slowest_time_and_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, total, ms, value in res:
        assert total == 15.0
        assert ms == 3.0
        assert abs(value - 2 * 1e12 / 3e-3 / 1e12) < 1e-9   # 2 replicas / 3 ms
