"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, spawned.

The path shards without an exchange (replicas), so the ranks only meet in a
barrier around the timed region and in the max-reduction of the step time;
the whole-job value counts every rank's bytes over the slowest rank's time.
The reference arm does its work on rank 0 alone.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    r, w, dist = bench.init_ranks("gloo", timeout_s=60)
    try:
        assert (r, w) == (rank, world)
        dist.barrier()
        ms = 1.5 + rank                       # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        value = bench.job_value(w, 4096e6, slowest)
        # the reference arm: rank 0 works, every other rank returns at once
        args = bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "0"])
        ref = bench.run_reference(args, r) if r != 0 else None
        dist.barrier()
        out[rank] = (slowest, value, ref is None)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_and_value_counts_all_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0, 0], codes
        res = dict(out)
    for r in range(world):
        slowest, value, ref_none = res[r]
        assert slowest == 2.5                                   # max over ranks, on every rank
        assert value == pytest.approx(world * 4096e6 / 2.5e-3 / 1e9)
        assert ref_none
    assert torch.distributed.is_available()


def test_single_rank_needs_no_process_group(monkeypatch):
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    sys.path.insert(0, ROOT)
    import bench
    rank, world, dist = bench.init_ranks("gloo")
    assert (rank, world, dist) == (0, 1, None)
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.job_value(1, 1e9, 1000.0) == pytest.approx(1.0)
