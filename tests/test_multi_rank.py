"""The multi-GPU path is replicas only: every rank runs the whole decode path on its own
cache, and the only cross-rank steps are the barrier and the max-over-ranks timing that
bench.py uses.  These run as world_size-2 gloo ranks on the CPU."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # each rank measured a different step time; all must report the slowest
        ms = bench.max_over_ranks(torch, dist, 2.0 + rank)
        dist.barrier()
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 3.0, 1: 3.0}


def test_single_process_timing_is_unchanged():
    assert bench.max_over_ranks(torch, None, 1.25) == 1.25


@pytest.mark.parametrize("world", [1, 2, 8])
def test_aggregate_value_is_whole_job_weak_scaling(world):
    # N replicas each stream the same bytes; the slowest rank's step time counts
    assert bench.aggregate_value(world, 1e9, 1.0) == pytest.approx(world * 1000.0)
