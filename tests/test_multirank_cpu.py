"""The N>1 plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path shards by (batch, head) with no exchange step, so `bench.py --gpus N` runs N replicas
and only reduces timings: each rank times its own steps, the job's time is the max over ranks,
and the whole-job throughput counts the work of every rank.  These tests run that reduction in
real processes (world size 2, gloo backend) and check the reference arm's rank handling."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out_q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], dist, "cpu")
        dist.barrier()
        out_q.put((rank, ms, bench.job_throughput(1e12, world, 10, ms)))
    finally:
        dist.destroy_process_group()


def test_job_time_is_the_slowest_rank_and_throughput_counts_all_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, times = 2, [3.0, 5.0]
    port = free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, tflops in got:
        assert ms == 5.0                                   # every rank sees the max
        assert tflops == pytest.approx(1e12 * 2 * 10 / 5e-3 / 1e12)


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.job_throughput(2e12, 1, 4, 8.0) == pytest.approx(1000.0)


@pytest.mark.parametrize("rank", ["1"])
def test_reference_arm_non_zero_rank_exits_without_work(rank):
    env = dict(os.environ, RANK=rank, WORLD_SIZE="2", LOCAL_RANK=rank)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "1",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True
