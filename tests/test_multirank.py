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


# ------------------------------------------------ one problem split by heads

def test_head_ranges_partition_every_head_exactly_once():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    for heads in (1, 2, 7, 8, 12, 32, 96, 256):
        for world in (1, 2, 3, 4, 8):
            if heads < world:
                with pytest.raises(ValueError):
                    bench.head_range(heads, world, 0)
                continue
            ranges = [bench.head_range(heads, world, r) for r in range(world)]
            covered = [h for a, b in ranges for h in range(a, b)]
            assert covered == list(range(heads)), (heads, world, ranges)
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_head_slices_are_the_heads_of_the_full_problem():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads
    w = workloads.Workload("t", 2, 3, 40, 8, "block", 0.3)
    x = workloads.make_inputs(w, 4)
    parts = [bench.slice_heads(x, w, *bench.head_range(6, 4, r)) for r in range(4)]
    for n in ("Q", "K", "V", "dO"):
        joined = torch.cat([p[n].reshape(-1, w.N, w.d) for p in parts])
        assert torch.equal(joined, x[n].reshape(6, w.N, w.d))
        assert all(p[n].is_contiguous() and p[n].shape[0] == 1 for p in parts)
    assert all(torch.equal(p["mask"], x["mask"]) for p in parts)


def _split_rank(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    h0, h1 = bench.head_range(32, world, rank)
    got = [None] * world
    dist.all_gather_object(got, (h0, h1))
    local_ms = 4.0 + rank                  # rank 1 is the slow one
    total = bench.max_over_ranks(local_ms, dist)
    ms, value = bench.throughput(total, steps=2, world=1, flops_per_step=1e12)  # one problem
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, total, ms, value))


def test_two_ranks_split_one_problem_by_heads():
    """The head split on two gloo ranks: both see the same partition of the
    32 heads, and the job's throughput is the one problem's work over the
    slowest rank's time (no factor of N)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, total, ms, value in res:
        assert got == [(0, 16), (16, 32)]
        assert total == 5.0 and ms == 2.5
        assert abs(value - 1e12 / 2.5e-3 / 1e12) < 1e-9
