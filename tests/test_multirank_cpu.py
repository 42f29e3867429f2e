"""The multi-GPU path of bench.py on the CPU: the split of the (batch, kv head)
units across ranks, and, with the gloo backend at world size 2, the max over
ranks, the all-gather that assembles the split outputs, and the reference arm
running on rank 0 only."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_unit_ranges_cover_every_unit_once():
    for units in range(1, 41):
        for world in range(1, 11):
            ranges = [bench.unit_range(units, world, k) for k in range(world)]
            flat = [u for lo, hi in ranges for u in range(lo, hi)]
            assert flat == list(range(units))                       # every unit once, in order
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1                      # balanced (uneven U / N too)


SMALL = WORKLOADS["kv"].replace(batch=2, hq=6, hkv=3, n_k=64, n_q=5, d=8, dv=8, r=4)


def test_strong_split_slices_one_draw_of_the_workload():
    Q, K, V = make_inputs(SMALL, seed=7)
    U, group = SMALL.batch * SMALL.hkv, SMALL.hq // SMALL.hkv
    world = 4                                                      # 6 units over 4 ranks: 1, 2, 1, 2
    parts = [bench.local_problem(SMALL, 7, world, k, "strong") for k in range(world)]
    assert [p[4] for p in parts] == [bench.unit_range(U, world, k)[0] for k in range(world)]   # unit_base
    assert all(p[5] == SMALL.batch * SMALL.n_q for p in parts)     # the whole job's tokens
    Kc = torch.cat([p[1] for p in parts])                          # [U, 1, n, d]
    Qc = torch.cat([p[0] for p in parts])                          # [U, group, nq, d]
    Vc = torch.cat([p[2] for p in parts])
    assert torch.equal(Kc.reshape(K.shape), K) and torch.equal(Vc.reshape(V.shape), V)
    # query head g of batch b reads kv head g // group: unit b * hkv + g // group
    for b in range(SMALL.batch):
        for g in range(SMALL.hq):
            assert torch.equal(Qc[b * SMALL.hkv + g // group, g % group], Q[b, g])
    wl = parts[1][3]
    assert (wl.batch, wl.hq, wl.hkv) == (2, group, 1)


def test_weak_split_stacks_workloads_with_distinct_units():
    world, U = 3, SMALL.batch * SMALL.hkv
    parts = [bench.local_problem(SMALL, 7, world, k, "weak") for k in range(world)]
    assert [p[4] for p in parts] == [0, U, 2 * U]                 # unit_base: blocks of one stack
    assert all(p[3] == SMALL and p[5] == world * SMALL.batch * SMALL.n_q for p in parts)
    assert not torch.equal(parts[0][1], parts[1][1])              # distinct batch blocks
    Q0, K0, V0 = make_inputs(SMALL, seed=7)
    assert torch.equal(parts[0][1], K0)                            # block 0 is the workload's own draw


def test_strong_split_needs_a_unit_per_rank():
    with pytest.raises(SystemExit):
        bench.local_problem(WORKLOADS["tiny"], 0, 2, 0, "strong")   # 1 unit: rank 0 gets none


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        w, r, _ = bench.dist_setup(world)
        assert (w, r) == (world, rank)
        local_ms = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(local_ms, w)
        bench.barrier(w)
        # stub outputs of a strong split of 5 units: each unit's block holds its unit index
        U = 5
        lo, hi = bench.unit_range(U, w, r)
        out = torch.arange(lo, hi, dtype=torch.float32).reshape(-1, 1, 1, 1).expand(-1, 2, 3, 4).contiguous()
        full = bench.gather_units(out, U, w, r)

        # the reference arm runs on rank 0 only; other ranks return without work
        class A:
            workload, warmup, steps, seed, ref_pivots, bins, center = "tiny", 0, 1, 0, 8, 1, False
            scaling, ref_budget_s = "weak", 60.0
        ref = bench.run_reference(A, w, r)
        q.put((rank, slowest, full.numpy().tolist(), None if ref is None else ref["impl"]))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_max_time_gather_and_reference():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    want = torch.arange(5, dtype=torch.float32).reshape(-1, 1, 1, 1).expand(-1, 2, 3, 4)
    for rank, slowest, full, ref in res:
        assert slowest == 15.0                                     # max over ranks
        assert torch.equal(torch.tensor(full), want)               # = the single-rank assembly
        assert ref == ("reference" if rank == 0 else None)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.shard_seed(7, 0) == 7
    assert bench.unit_range(8, 1, 0) == (0, 8)
