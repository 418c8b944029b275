"""Multi-rank logic of bench.py on CPU: two gloo ranks, and the reference arm's rank rule.

bench.py times each rank on its own device and reports the whole job as the
units of all ranks over the slowest rank's time; the reference arm (the oracle
on the host) runs on rank 0 only.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_seconds, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(local_seconds[rank], world, "cpu")
        queue.put((rank, t, bench.job_throughput(32, world, t)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_slowest_time_and_whole_job_rate():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    local_seconds = [0.5, 0.8]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, local_seconds, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in results:
        assert t == 0.8                      # both ranks see the slowest rank's time
        assert v == pytest.approx(2 * 32 / 0.8)


def _run_reference(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--gpus", "2", "--steps", "3", "--warmup", "3", "--oracle-budget", "0.2"]
    return subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _run_reference(1)
    assert r1.returncode == 0, r1.stderr
    assert r1.stdout.strip() == ""
    r0 = _run_reference(0)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
