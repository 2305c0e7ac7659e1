"""The multi-GPU path is replicas only: every rank runs its own batch, with no
collective on the data path; the bench takes the slowest rank's time and the
whole job's units.  These run that host logic as two gloo ranks on the CPU."""

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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.ranks_from_env()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, w, torch.device("cpu"))
        rate = bench.whole_job_rate(w, 256, 20, ms / 1e3)
        out[rank] = (r, w, local, ms, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank_and_the_whole_job():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    for rank in range(world):
        r, w, local, ms, rate = res[rank]
        assert (r, w, local) == (rank, world, rank)
        assert ms == pytest.approx(15.0)                     # the max over ranks, on every rank
        assert rate == pytest.approx(2 * 256 * 20 / 0.015)   # both ranks' chunks over the slowest time


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.whole_job_rate(1, 256, 10, 2.0) == pytest.approx(1280.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    """Under torchrun the oracle arm runs on rank 0; other ranks exit without work."""
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps = 1
        warmup = 0
        gpus = 2

    assert bench.run_reference(Args(), rank=1) is None
    assert capsys.readouterr().out == ""
