"""Host-side logic of the multi-GPU (replicas) path of bench.py, run as 2 gloo ranks on the CPU.

The forward does not shard (one batch-1 forward is a chain of 25 coupled blocks), so N GPUs
run N independent replicas; the only collectives are a barrier and a max over ranks of the
timed region.  These tests exercise exactly those pieces without a GPU.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # each rank timed its own replicas; the whole job is as slow as the slowest rank
        ms = 100.0 + 25.0 * rank
        mx = bench.max_over_ranks(ms, world)
        value = bench.aggregate_ms_per_forward(mx, 4, world)
        assert bench.dist_env() == (world, rank, rank)
        # the reference arm runs on rank 0 only; other ranks return at once without work
        class A:
            steps, warmup, gpus = 1, 3, world
        rc = bench.run_reference(A, None) if rank != 0 else 0
        bench.barrier(world)
        out.put((rank, mx, value, rc))
    finally:
        dist.destroy_process_group()


def test_replica_timing_max_and_aggregate_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, value, rc in res:
        assert mx == 125.0                       # max over ranks, seen by every rank
        assert value == 125.0 / (4 * world)      # whole-job ms per forward
        assert rc == 0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_ms_per_forward(200.0, 20, 1) == 10.0


def test_reference_arm_prints_one_json_line_on_the_cpu():
    """bench.py --impl reference times the CPU oracle; tiny workload so it ends in seconds."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny64",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "ms/forward" and j["higher_is_better"] is False
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0
    assert j["value"] > 0
