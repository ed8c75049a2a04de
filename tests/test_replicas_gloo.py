"""The multi-GPU path is replicas only: every rank runs the whole workload on
its own GPU, nothing is exchanged, and the job's time is the slowest rank's.
The host logic of that path runs here on CPU ranks over gloo (world size 2):
the max-over-ranks reduction and the weak-scaling throughput bench.py
reports, and the reference arm under torchrun, where rank 0 alone works and
prints one line and the other ranks exit 0."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        q.put((rank, bench.reduce_max(ms, dist, "cpu")))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_is_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 15.0, 1: 15.0}


def test_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas x 32768 timesteps per step x 10 steps in 100 ms
    assert bench.job_throughput(2, 32768, 10, 100.0) == pytest.approx(6_553_600.0)
    assert bench.job_throughput(1, 32768, 10, 100.0) == pytest.approx(3_276_800.0)
    assert bench.reduce_max(3.5) == 3.5  # one process: no group, the value itself


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "1", "--workload", "lstm_T8_B2_I16_H32_fp32"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout  # rank 0 alone prints
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
