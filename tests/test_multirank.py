"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks.

Every rank quantizes its own weight set (weak scaling, no data-path
collective); the step time is the maximum over ranks."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mats = bench.workload("llama2-70b", rank)
        labels = [m[0] for m in mats]
        streams = [(m[4], m[5]) for m in mats]
        # each rank's fake timing: rank-dependent values, reduced to the max
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank], dist)
        obj = [None] * world
        dist.all_gather_object(obj, (labels, streams, mx))
        if rank == 0:
            out.put(obj)
    finally:
        dist.destroy_process_group()


def test_two_ranks_disjoint_shards_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (l0, s0, m0), (l1, s1, m1) = res
    assert len(l0) == len(l1) == 560                    # same work per rank (weak scaling)
    assert not set(l0) & set(l1)                        # disjoint layers
    assert not set(s0) & set(s1)                        # distinct generator streams
    assert m0 == m1 == [11.0, 5.0]                      # max over ranks on every rank


def test_single_rank_max_is_identity():
    assert bench.max_over_ranks([3.0, 4.0], None) == [3.0, 4.0]
