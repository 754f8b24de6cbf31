"""The multi-process path of bench.py on CPU ranks (gloo, world size 2).

Decode is sharded by sequence replicas with no collective on the data path:
each rank draws and times its own caches, and the only cross-rank step is
taking the slowest rank's time. These tests run that step, the per-rank seed
split and the reference arm's rank-0-only rule on two gloo processes.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (10 + r) ms for the step loop and (5 - r) ms for the decode calls
        got = bench.cross_rank_max([10.0 + rank, 5.0 - rank], world, torch.device("cpu"))
        seeds = [bench.replica_seed(rank, r) for r in range(4)]
        ref = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})()) if rank == 1 else "skipped"
        q.put((rank, got, seeds, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_split_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict()
    for _ in procs:
        rank, got, seeds, ref = q.get(timeout=120)
        res[rank] = (got, seeds, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        assert res[rank][0] == [11.0, 5.0]  # max over ranks, seen by every rank
    assert not set(res[0][1]) & set(res[1][1])  # disjoint replica seeds
    assert res[1][2] is None  # the reference arm runs on rank 0 only


def test_single_rank_needs_no_collective():
    assert bench.cross_rank_max([3.0, 4.0], 1, None) == [3.0, 4.0]
