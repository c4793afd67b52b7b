"""The multi-GPU bench path on CPU: two gloo ranks, replicas with no data-path
collective; the timing is the max over ranks and the value the whole-job rate."""
import datetime
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference (the fp64 oracle on the host cores) runs without a GPU and prints the
    JSON line the driver compares against."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "seq-steps/s" and d["value"] > 0 and d["higher_is_better"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_bench_byte_variants():
    """Page-rounded K/V bytes and the split partials' bytes that the bench line reports beside the
    algorithmic bytes (bench-side arithmetic, no GPU)."""
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.DecodeConfig("t", "bf16", B=2, H_q=8, H_kv=2, Dh=128, page_size=16)
    lens = [17, 32]  # 2 and 2 pages
    v = bench.kv_byte_variants(cfg, lens, 2, 2, S=1, C=0)
    assert v["kv_bytes_page_rounded"] == 4 * 16 * 2 * 128 * 2 * 2 and v["partials_bytes_write_read"] == 0
    # grid split of 2 splits, 1 page each: every row fills both splits -> 2 partials per (row, KV head)
    v = bench.kv_byte_variants(cfg, lens, 2, 2, S=2, C=1)
    assert v["partials_bytes_write_read"] == 2 * (2 * 2 * 2) * 4 * (128 + 2) * 4
    # planned chunks of 2 pages: each row has one chunk -> no partials
    assert bench.kv_byte_variants(cfg, lens, 2, 2, S=0, C=0, plan_C=2)["partials_bytes_write_read"] == 0
    f = bench.roofline_fracs(4000.0, 8000.0)
    assert f["frac"] == 0.5 and f["frac_datasheet"] == 0.5
