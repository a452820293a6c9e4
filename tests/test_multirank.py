"""The N > 1 path of bench.py on CPU: two gloo ranks (one process each) run
the same cross-rank step the GPU replicas run over NCCL -- the slowest rank's
time becomes the job's time on every rank, and the whole-job value counts
every rank's units -- and the reference arm does its work on rank 0 only."""
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


def _rank(rank, world, port, times, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms_max = bench.max_over_ranks(times[rank], "cpu", world)
        out[rank] = (ms_max, bench.whole_job_value(world, 1e12, ms_max))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_value(world):
    times = [3.0, 5.0]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, world, port, times, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        got = dict(out)
    for r in range(world):
        ms_max, value = got[r]
        assert ms_max == 5.0
        assert abs(value - world * 1e12 / 5e-3 / 1e12) < 1e-9   # 400 (1e12 units per rank, 5 ms)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, "cpu", 1) == 2.5
    assert bench.whole_job_value(1, 2e12, 2.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, gpus = 1, 3, 2
    assert bench.run_reference(Args(), bench.WORKLOADS["tiny_fp32"]) == 0   # returns without any work
