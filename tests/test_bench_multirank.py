"""The N > 1 bookkeeping of bench.py on CPU: two gloo ranks (world size 2, 127.0.0.1).

A multi-GPU run gives every rank its own sequence (weak scaling) and reports the whole job's
throughput against the slowest rank's time; only rank 0 prints, and the reference arm does its
work on rank 0 alone.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        import bench
        ms, value = bench.job_throughput(10.0 + 5.0 * rank, 1024, 20, world, "cpu")
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_and_all_tokens():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in got:
        assert ms == 15.0                                    # max over ranks, on every rank
        assert value == pytest.approx(1024 * 20 * 2 / 0.015)  # both ranks' tokens


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.job_throughput(8.0, 1024, 10, 1, "cpu")
    assert ms == 8.0 and value == pytest.approx(1024 * 10 / 0.008)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
