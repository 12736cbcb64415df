"""The N > 1 path of bench.py on CPU: two gloo ranks (one process each, 127.0.0.1) take the
timing reduction and the whole-job value of the replicas-only scaling, and the reference
arm runs on rank 0 alone. No GPU: the path shards into independent replicas with no data
exchange, so the collective under test is the max-over-ranks of the timing."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        reduce = bench.max_over_ranks_fn(torch, dist, world, torch.device("cpu"))
        local_ms = [0.120, 0.135][rank]                 # rank 1 is the slowest
        ms = reduce(local_ms)
        value = bench.replica_value(world, 561512448, ms)
        # the reference arm prints (and works) on rank 0 only; other ranks return at once
        args = type("A", (), {"steps": 1, "warmup": 0, "batch": 1, "ref_rows": 1})()
        returned_early = None
        if rank != 0:
            bench.run_reference(args)
            returned_early = True
        q.put((rank, ms, value, returned_early))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_scale_weakly():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value, early in got:
        assert ms == pytest.approx(0.135)                # every rank sees the max
        assert value == pytest.approx(2 * 561512448 / 0.135e-3 / 1e9)
        assert early is (True if rank == 1 else None)


def test_single_rank_values():
    sys.path.insert(0, ROOT)
    import bench
    reduce = bench.max_over_ranks_fn(torch, dist, 1, torch.device("cpu"))
    assert reduce(0.5) == 0.5
    assert bench.replica_value(1, 10**9, 1000.0) == pytest.approx(1.0)
