"""Multi-rank host logic of bench.py on CPU: gloo, world size 2.

The GPU path shards by replicas with no data-path collective; what the ranks
share is the barrier and the max over ranks of the timed interval, exercised
here with gloo in two processes.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank               # rank 1 is the slow one
        got = bench.max_over_ranks(ms, torch.device("cpu"), world)
        # per-sample maxima: each rank is the slow one on some samples
        samples = [1.0, 2.0, 3.0] if rank == 0 else [3.0, 1.0, 2.5]
        per = bench.max_over_ranks_all(samples, torch.device("cpu"), world)
        q.put((rank, got, bench.job_throughput(1_000_000, 100, got, world), per))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    assert [r[3] for r in res] == [[3.0, 2.0, 3.0]] * 2
    # 2 ranks x 100 steps x 1 MB over 15 ms
    assert abs(res[0][2] - 2 * 100 * 1e6 / 15e-3 / 1e9) < 1e-9


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, None, 1) == 3.5
    assert bench.max_over_ranks_all([3.5, 1.0], None, 1) == [3.5, 1.0]
    assert abs(bench.job_throughput(176_619_520, 1, 0.027, 1) - 6541.46) < 0.01


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3", "--workload", "masked_decode"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "3", "--warmup", "3", "--workload", "masked_decode"],
                         env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    lines = res.stdout.strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
