"""The multi-GPU bench path on CPU: two gloo ranks, replicas with no data-path
collective; the timing is the max over ranks and the value the whole-job rate."""
import datetime
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from paged_kv_cache_433_b200 import workloads as W

        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(elapsed, world)
        bench.barrier(world)
        order = W.page_order(1000, W.LLAMA8B.seed + 1000 * rank)  # each replica shuffles its own pool
        q.put((rank, m, bench.replica_value(64, 100, world, m), order[:8].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, o0), (r1, m1, v1, o1) = res
    assert m0 == m1 == 15.0
    assert v0 == v1 == pytest.approx(64 * 100 * 2 / 0.015)
    assert o0 != o1
