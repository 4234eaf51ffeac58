"""World-size-2 checks of the benchmark's multi-rank host logic on CPU (gloo): the timed region's
max over ranks, the whole-job rate, per-rank inputs, and the reference arm's rank gating."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [10.0, 13.5][rank]
        ms = bench.reduce_max(local_ms, world, torch.device("cpu"))
        rate = bench.whole_job_rate(world, 32760, 20, ms)
        seed = bench.rank_seed_base(2000, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        dist.barrier()
        q.put((rank, ms, rate, seeds))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_rate_on_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, rate, seeds in res:
        assert ms == 13.5                       # the slowest rank's time
        assert rate == pytest.approx(2 * 32760 * 20 / 0.0135)
        assert len(set(seeds)) == world          # every rank draws its own sequences


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup = 1, 0
    assert bench.run_reference(A()) == 0        # exits without work on ranks other than 0
