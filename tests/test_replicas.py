"""The multi-GPU form of the benchmark is replicas only: every rank streams its own copy of the
stack, and the job's figure is all ranks' bytes over the slowest rank's device time. These
tests run that host logic as world-size-2 `gloo` process groups on the CPU."""

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
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (10 + r) ms for its passes and (20 - r) ms end to end
        total_ms, e2e_ms = bench.max_over_ranks([10.0 + rank, 20.0 - rank], "cpu", world)
        q.put((rank, total_ms, e2e_ms, bench.job_gbs(world, 1e9, total_ms)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total_ms, e2e_ms, gbs in results:
        assert total_ms == 11.0 and e2e_ms == 20.0          # the slowest rank's times, on every rank
        assert gbs == pytest.approx(2 * 1e9 / 11e-3 / 1e9)  # both ranks' bytes over that time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], "cpu", 1) == [3.0, 4.0]
    assert bench.job_gbs(1, 2e9, 1000.0) == pytest.approx(2.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "cpu_sample", lambda *a, **k: called.append(1))
    args = argparse.Namespace(gpus=2, steps=1, warmup=3, impl="reference")
    assert bench.run_reference(args) == 0
    assert not called
