"""The split of one problem's (batch, kv head) units across GPUs, run on one
GPU as separate calls: each call holds a block of units and passes the index
of its first unit as unit_base, so every unit draws the pivots it draws in one
call over the whole problem.  Pivots and ranks must match that call exactly,
the outputs to 1e-5 of their largest entry (the calls differ only in launch
plans: key blocks per unit, attention splits)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import bench
from coreset_attention_approximation_b200 import wildcat
from coreset_attention_approximation_b200.workloads import WORKLOADS
from parity import rel_err

pytestmark = pytest.mark.gpu

W = WORKLOADS["kv"].replace(batch=2, hq=8, hkv=2, n_k=4096, n_q=200, r=128)


def _run(Q, K, V, r, **kw):
    res = wildcat.forward(Q.cuda(), K.cuda(), V.cuda(), r, seed=3, **kw)
    torch.cuda.synchronize()
    assert wildcat.check_device_status(res["ws"]) == 0
    return {k: v.cpu() for k, v in res.items() if k != "ws"}


@pytest.mark.parametrize("bins", [1, 2])
def test_strong_split_matches_one_call(bins):
    U, group = W.batch * W.hkv, W.hq // W.hkv
    Q, K, V, _, _, _ = bench.local_problem(W, 3, 1, 0, "strong")
    full = _run(Q, K, V, W.r, bins=bins)
    piv = full["piv"].reshape(U, W.r)
    rank = full["rank"].reshape(U, -1)
    out = full["out"].reshape(U, group, W.n_q, W.dv)
    for world in (3, 4):                                  # 4 units: uneven (1, 1, 2) and one per call
        for k in range(world):
            Qk, Kk, Vk, wl, base, _ = bench.local_problem(W, 3, world, k, "strong")
            part = _run(Qk, Kk, Vk, W.r, bins=bins, unit_base=base)
            n = wl.batch
            assert torch.equal(part["piv"].reshape(n, W.r), piv[base:base + n])
            assert torch.equal(part["rank"].reshape(n, -1), rank[base:base + n])
            got = part["out"].reshape(n, group, W.n_q, W.dv)
            for u in range(n):
                assert rel_err(got[u].numpy(), out[base + u].numpy()) <= 1e-5


def test_weak_split_matches_one_call_over_the_stack():
    world, U = 2, W.batch * W.hkv
    parts = [bench.local_problem(W, 3, world, k, "weak") for k in range(world)]
    stack = [torch.cat([p[i] for p in parts]) for i in range(3)]          # batch world * B
    full = _run(*stack, W.r)
    for k, (Qk, Kk, Vk, wl, base, _) in enumerate(parts):
        assert base == k * U
        part = _run(Qk, Kk, Vk, W.r, unit_base=base)
        assert torch.equal(part["piv"], full["piv"][k * W.batch:(k + 1) * W.batch])
        for b in range(W.batch):
            for h in range(W.hq):
                assert rel_err(part["out"][b, h].numpy(), full["out"][k * W.batch + b, h].numpy()) <= 1e-5


def test_unit_base_changes_the_draws():
    Q, K, V, _, _, _ = bench.local_problem(W, 3, 1, 0, "strong")
    a = _run(Q, K, V, W.r)["piv"].numpy()
    b = _run(Q, K, V, W.r, unit_base=5)["piv"].numpy()
    assert not np.array_equal(a, b)


def _select_kernels(K, r, **kw):
    import re
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        wildcat.select(K.cuda(), r, seed=3, **kw)
        torch.cuda.synchronize()
    return {m.group(0) for e in prof.events() if e.device_type.name == "CUDA"
            for m in [re.search(r"rpcholesky_\w*kernel", e.name)] if m}


def test_strong_split_across_select_forms():
    # 160 short heads: one block per unit in one call; 80 per part, fewer than
    # the SMs, take a cluster per unit.  The pivots do not depend on the form;
    # the outputs agree to the bf16 path's tolerance, since the attention and
    # weights GEMMs also split their work by the head count (fp16 P rounded
    # against other running maxima, partial sums merged in another order).
    w = WORKLOADS["vit"].replace(batch=2, hq=80, hkv=80, n_q=64)
    U, group = w.batch * w.hkv, w.hq // w.hkv
    Q, K, V, _, _, _ = bench.local_problem(w, 3, 1, 0, "strong")
    full = _run(Q, K, V, w.r)
    kinds = {frozenset(_select_kernels(K, w.r))}
    piv = full["piv"].reshape(U, w.r)
    out = full["out"].reshape(U, group, w.n_q, w.dv)
    for k in range(2):
        Qk, Kk, Vk, wl, base, _ = bench.local_problem(w, 3, 2, k, "strong")
        kinds.add(frozenset(_select_kernels(Kk, w.r, unit_base=base)))
        part = _run(Qk, Kk, Vk, w.r, unit_base=base)
        n = wl.batch
        assert torch.equal(part["piv"].reshape(n, w.r), piv[base:base + n])
        got = part["out"].reshape(n, group, w.n_q, w.dv)
        for u in range(n):
            assert rel_err(got[u].numpy(), out[base + u].numpy()) <= 2e-3
    assert kinds == {frozenset({"rpcholesky_unit_kernel"}), frozenset({"rpcholesky_cluster_kernel"})}
