"""The multi-rank plumbing of bench.py on the CPU.

bench.py runs one process per GPU under torchrun; the path does not shard, so N ranks are N
independent replicas, timed on the device and aggregated as max-over-ranks time and the
whole job's units.  Here two gloo ranks (spawned processes, 127.0.0.1 rendezvous) go through
the same helpers: joining the group, the max over ranks of a rank-dependent time, the
barrier and the whole-job throughput; and the reference arm does its work on rank 0 only.
"""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, _ = bench.dist_setup(world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * r, w)  # rank r took 10 + 5 r ms
        bench.barrier(w)
        q.put((r, w, ms, bench.job_throughput(100, 4, w, ms), dist.get_backend()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_the_whole_jobs_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r for r, *_ in res] == [0, 1]
    for _, w, ms, v, backend in res:
        assert w == 2 and backend == "gloo"
        assert ms == 15.0  # every rank reports the slowest rank's time
        assert v == pytest.approx(100 * 4 * 2 / 15e-3)  # units of both replicas over that time


def test_job_throughput_single_rank():
    import bench
    assert bench.job_throughput(2048, 3, 1, 30.0) == pytest.approx(2048 * 3 / 0.03)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert rc == 0 and out.getvalue() == ""
