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


def _shard_worker(rank, world, port, out):
    """Rank `rank` runs the oracle on its rows of a global batch of the tiny
    workload and gathers every rank's actions."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    import bench
    import oracle
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.workload("tiny", batch=5, fixed_ids=(1, 0, 0, 1, 1), valid_min=20)
        W = synth.make_weights(w.geom)
        inp = synth.make_inputs(w, seed=3)
        a, b = bench.shard_rows(w.batch, rank, world)
        mine = oracle.get_action(W, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"],
                                 inp["embodiment_id"], inp["init_noise"], w.num_steps, samples=range(a, b))
        got = bench.gather_rows(torch.from_numpy(np.ascontiguousarray(mine)), w.batch, world)
        out[rank] = got.numpy().tobytes()
    finally:
        dist.destroy_process_group()


def test_batch_sharded_ranks_gather_the_single_process_result():
    """A global batch of 5 split over 2 ranks (3 + 2 rows), each rank's slice
    through the oracle, gathered: bit-identical to one process running all 5."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    import synth
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    w = synth.workload("tiny", batch=5, fixed_ids=(1, 0, 0, 1, 1), valid_min=20)
    W = synth.make_weights(w.geom)
    inp = synth.make_inputs(w, seed=3)
    whole = oracle.get_action(W, w.geom, inp["backbone_features"], inp["vl_mask"], inp["state"],
                              inp["embodiment_id"], inp["init_noise"], w.num_steps)
    for rank in range(world):
        got = np.frombuffer(res[rank], dtype=whole.dtype).reshape(whole.shape)
        np.testing.assert_array_equal(got, whole)


def test_shard_rows_cover_the_batch_once():
    sys.path.insert(0, ROOT)
    import bench
    for B in (1, 5, 8, 256, 257):
        for world in (1, 2, 3, 8):
            spans = [bench.shard_rows(B, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(spans[r][1] == spans[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


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
