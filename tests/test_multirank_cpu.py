"""Multi-rank host logic of bench.py on the CPU: two gloo ranks.

The layer runs as independent replicas (one per GPU, no collective on the data
path); what is shared between ranks is the timing: every rank's step time is
reduced with a max, and the whole-job throughput counts every rank's work over
the slowest rank's time. The reference arm runs on rank 0 only.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r reports step times (r + 1, 5 - r) ms: the job sees the slowest rank's
        got = bench.max_over_ranks(dist, torch.device("cpu"), rank + 1.0, 5.0 - rank)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == [2.0, 5.0] and res[1] == [2.0, 5.0]


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench

    # 2 ranks x 1e12 FLOP each in 1000 ms (the slowest rank) = 2 TFLOP/s
    assert bench.job_throughput(2, 1e12, 1000.0) == pytest.approx(2.0)
    assert bench.job_throughput(1, 6.594e12, 0.87) == pytest.approx(6.594e12 / 0.87e-3 / 1e12)
    assert bench.max_over_ranks(None, None, 1.5, 2) == [1.5, 2.0]


@pytest.mark.timeout(120)
def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=110)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
