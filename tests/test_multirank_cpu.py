"""The multi-GPU path of bench.py, on CPU with the gloo backend, world size 2.

Every rank runs its own copy of the workload (independent (batch, kv-head)
units: no collective on the data path), the step time is the max over ranks,
and only rank 0 prints.  These tests run those pieces in two processes."""

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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        w, r, _ = bench.dist_setup(world)
        assert (w, r) == (world, rank)
        local_ms = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(local_ms, w)
        bench.barrier(w)
        seeds = [None] * w
        dist.all_gather_object(seeds, bench.shard_seed(0, r))
        # the reference arm runs on rank 0 only; other ranks return without work
        class A:
            workload, warmup, steps, seed, ref_pivots = "tiny", 0, 0, 0, 8
        ref = bench.run_reference(A, w, r) if r != 0 else "rank0"
        q.put((rank, slowest, seeds, ref))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_max_time_distinct_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, seeds, ref in res:
        assert slowest == 15.0                       # max over ranks
        assert len(set(seeds)) == 2                  # each rank draws its own inputs
        assert ref == ("rank0" if rank == 0 else None)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.shard_seed(7, 0) == 7
