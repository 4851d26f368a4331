"""The benchmark's multi-rank plumbing on CPU with the gloo backend, world size 2: every
rank gets the slowest rank's time, the job value counts every rank's tokens over that
time, and the reference arm does its work on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = [12.5, 20.0][rank]
        mx = bench.max_over_ranks(my_ms, world, device="cpu")
        value = bench.job_tokens_per_s(4096, world, 10, mx)
        dist.barrier()
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [20.0, 20.0]
    assert all(abs(g[2] - 4096 * 2 * 10 / 0.020) < 1e-6 for g in got)


def test_reference_arm_does_no_work_off_rank_0(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup, ref_step_s = "decode1", 1, 3, 1.0

    assert bench.run_reference(A(), world=2, rank=1) is None
