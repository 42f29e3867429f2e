"""GPU parity of the binned selection (the method's divide-and-conquer
selection, WildCat gist.science summary "Methodik" item 1 "Effizienz") and of
key centring ("Methodik" item 3) against the oracle, through the C ABI."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from parity import TOL_OUT, compare_next, rel_err, run_gpu
import oracle
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_bins_tiny_fp32():
    w = WORKLOADS["tiny"]
    compare_next(*make_inputs(w), w.r, seed=0, bins=2, tol_w=1e-5)


def test_bins_vit():
    w = WORKLOADS["vit"].replace(batch=4)
    compare_next(*make_inputs(w), w.r, seed=1, bins=2, tol_w=2e-3)


def test_bins_diffusion_four_bins():
    w = WORKLOADS["diffusion"].replace(batch=1, hq=4, hkv=4)
    compare_next(*make_inputs(w), w.r, seed=2, bins=4, tol_w=2e-3)


def test_bins_kv_gqa_eight_bins():
    w = WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=8192, r=256)
    compare_next(*make_inputs(w), w.r, seed=3, bins=8, tol_w=2e-3)


def test_bins_one_equals_plain_path():
    w = WORKLOADS["vit"].replace(batch=2)
    Q, K, V = make_inputs(w)
    a = run_gpu(Q, K, V, w.r, seed=4)
    b = run_gpu(Q, K, V, w.r, seed=4, bins=1)
    for k in ("piv", "rank", "F", "W", "out"):
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bins_rank_deficient_bins_reproduce_exact_attention(dtype):
    # Each bin of 256 keys holds 5 distinct rows: the bins stop at rank 5, their
    # padded coreset rows carry zero weights, and the union is exact attention.
    g = torch.Generator().manual_seed(6)
    bins, nb, d = 4, 256, 64
    blocks = []
    for b in range(bins):
        distinct = torch.randn(5, d, generator=g, dtype=torch.float64) * 0.6
        blocks.append(distinct[torch.arange(nb) % 5])
    K = torch.cat(blocks).reshape(1, 1, bins * nb, d).to(dtype)
    Q = (torch.randn(1, 1, 200, d, generator=g, dtype=torch.float64) * 0.6).to(dtype)
    V = torch.randn(1, 1, bins * nb, d, generator=g, dtype=torch.float64).to(dtype)
    rep = compare_next(Q, K, V, 64, seed=5, bins=bins)
    res = run_gpu(Q, K, V, 64, seed=5, bins=bins)
    assert np.all(res["rank"].numpy() == 5)
    beta = oracle.default_beta(d)
    ref = oracle.exact_attention(Q[0, 0].double().numpy(), K[0, 0].double().numpy(), V[0, 0].double().numpy(), beta)
    assert rel_err(res["out"][0, 0].numpy(), ref) <= TOL_OUT[dtype], rep


def test_bins_invalid_shapes_are_refused():
    from coreset_attention_approximation_b200 import wildcat
    w = WORKLOADS["vit"].replace(batch=1)
    Q, K, V = [t.cuda() for t in make_inputs(w)]
    with pytest.raises(wildcat.WildcatError):
        wildcat.forward(Q, K, V, w.r, bins=3)          # n = 1024 is not a multiple of 3
    with pytest.raises(wildcat.WildcatError):
        wildcat.forward(Q, K, V, 66, bins=4)           # r = 66 is not a multiple of 4


def _offset(w, seed, shift):
    """The workload's inputs with one common vector added to every key (the
    case centring exists for: the kernel matrix changes, attention does not)."""
    Q, K, V = make_inputs(w, seed=seed)
    g = torch.Generator().manual_seed(seed + 100)
    c = torch.randn(K.shape[-1], generator=g, dtype=torch.float64) * shift
    return Q, (K.double() + c).to(K.dtype), V


def test_center_tiny_fp32():
    w = WORKLOADS["tiny"]
    compare_next(*_offset(w, 0, 0.5), w.r, seed=0, center=True, tol_w=1e-5)


def test_center_vit():
    w = WORKLOADS["vit"].replace(batch=4)
    compare_next(*_offset(w, 1, 0.3), w.r, seed=1, center=True, tol_w=2e-3)


def test_center_diffusion_mixture():
    w = WORKLOADS["diffusion"].replace(batch=1, hq=4, hkv=4)
    compare_next(*make_inputs(w), w.r, seed=2, center=True, tol_w=2e-3)


def test_center_with_bins_kv():
    w = WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=8192, r=256)
    compare_next(*_offset(w, 3, 0.2), w.r, seed=3, bins=4, center=True, tol_w=2e-3)


def test_center_changes_the_selection_but_not_exactness():
    # A large common key offset: without centring the kernel matrix is dominated
    # by the offset; with it the run matches the oracle on the centred keys and
    # the output still approximates the same attention.
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=2, n_k=512, n_q=64, r=64)
    Q, K, V = _offset(w, 4, 1.0)
    a = run_gpu(Q, K, V, w.r, seed=4, center=True)
    b = run_gpu(Q, K, V, w.r, seed=4)
    assert not torch.equal(a["piv"], b["piv"])
    compare_next(Q, K, V, w.r, seed=4, center=True, tol_w=2e-3)


def test_bins_without_queries_runs_select_and_weights():
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=2, n_q=0)
    Q, K, V = make_inputs(w)
    res = run_gpu(Q, K, V, w.r, seed=7, bins=4)
    assert res["rank"].shape == (1, 2, 4) and np.all(res["rank"].numpy() == w.r // 4)
    assert res["out"].numel() == 0


def test_bins_one_pivot_per_bin():
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=2, n_k=512, n_q=40, r=8)
    compare_next(*make_inputs(w, seed=8), 8, seed=8, bins=8, tol_w=2e-3)


def test_center_with_bins_fp32():
    w = WORKLOADS["tiny"]
    compare_next(*_offset(w, 9, 0.4), w.r, seed=9, bins=4, center=True, tol_w=1e-5)


def test_bins_attend_without_allocation():
    # the attention entry that allocates nothing takes every union row as well
    from coreset_attention_approximation_b200 import wildcat
    w = WORKLOADS["diffusion"].replace(batch=1, hq=2, hkv=2, n_k=2048, n_q=300, r=128)
    Q, K, V = [t.cuda() for t in make_inputs(w, seed=11)]
    res = wildcat.forward(Q, K, V, w.r, seed=11, bins=4)
    want = wildcat.attend(Q, res["Ks"], res["W"], res["rank"], w.n_k, bins=4)
    got = wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k, bins=4)
    torch.cuda.synchronize()
    assert wildcat.check_device_status(res["ws"]) == 0
    for h in range(w.hq):
        assert rel_err(got[0, h].cpu().numpy(), want[0, h].cpu().numpy()) <= TOL_OUT[torch.bfloat16]
        assert rel_err(got[0, h].cpu().numpy(), res["out"][0, h].cpu().numpy()) <= TOL_OUT[torch.bfloat16]
