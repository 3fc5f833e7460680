"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (no GPU).

Each rank runs its own sequence; the job time is the maximum over ranks and
the throughput counts every rank's tokens.  The oracle ("reference") arm runs
on rank 0 only; other ranks exit without work.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local = [3.0, 7.5][rank]            # per-rank device time in ms
    job = bench.max_over_ranks(local)
    thr = bench.job_throughput(world, 32760, 10, job)
    q.put((rank, job, thr))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
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
    for rank, job, thr in res:
        assert job == 7.5                                   # max over ranks, same on every rank
        assert thr == pytest.approx(2 * 32760 * 10 / 7.5e-3)


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.job_throughput(1, 100, 4, 2.0) == pytest.approx(200000.0)


def test_reference_arm_nonzero_rank_does_no_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 2, 1, 2
    assert bench.run_reference(A()) == 0
