"""The bounds-checked build (libwildcat_debug.so): the same results as the
release library on parity cases, and out-of-range pivots or ranks handed to
the weights and attention calls recorded as WC_ERR_BOUNDS instead of read.

Every read of a caller-supplied pivot or rank in those calls is guarded in this
build (gather, centred merge, solves, the exp-GEMMs, the weight preparation),
so the invalid inputs below never reach memory."""

import pytest
import torch

from coreset_attention_approximation_b200 import wildcat
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs
from parity import compare, compare_next

pytestmark = pytest.mark.gpu

BOUNDS = 7


@pytest.fixture
def debug_lib():
    wildcat.use_debug_library(True)
    try:
        yield
    finally:
        wildcat.use_debug_library(False)


def test_debug_build_matches_the_oracle(debug_lib):
    w = WORKLOADS["long"].replace(hq=4, hkv=2, n_k=8192, n_q=777, r=256)
    compare(*make_inputs(w, seed=31), w.r, seed=31, tol_w=2e-3)
    w = WORKLOADS["tiny"]
    compare(*make_inputs(w), w.r, seed=0, tol_w=1e-5)
    w = WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=4096, n_q=256, r=256)
    compare_next(*make_inputs(w, seed=32), w.r, seed=32, bins=4, center=True, tol_w=2e-3)
    # the select's forms for shorter units: one block per unit, a cluster per unit
    w = WORKLOADS["vit"].replace(batch=2, hq=80, hkv=80, n_q=128)
    compare(*make_inputs(w, seed=34), w.r, seed=34, tol_w=2e-3)
    w = WORKLOADS["diffusion"].replace(r=48, n_q=256)
    compare(*make_inputs(w, seed=35), w.r, seed=35, tol_w=2e-3)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_bad_pivots_and_ranks_are_recorded_not_read(debug_lib, dtype):
    w = WORKLOADS["vit"].replace(batch=1, hq=2, hkv=2, n_k=600, n_q=100, r=32,
                                 dtype="bf16" if dtype == torch.bfloat16 else "f32")
    Q, K, V = [t.cuda() for t in make_inputs(w, seed=33)]
    res = wildcat.forward(Q, K, V, w.r, seed=1)
    ws = res["ws"]
    assert wildcat.check_device_status(ws) == 0
    for bad in (w.n_k + 5, -7):
        piv = res["piv"].clone()
        piv[0, 1, 3] = bad
        wildcat.weights(K, V, piv, res["F"], res["rank"], w.r, ws=ws, seed=1)
        assert wildcat.check_device_status(ws) == BOUNDS
        assert wildcat.check_device_status(ws) == 0               # read and cleared
    rank = res["rank"].clone()
    rank[0, 0] = w.r + 3
    wildcat.weights(K, V, res["piv"], res["F"], rank, w.r, ws=ws, seed=1)
    assert wildcat.check_device_status(ws) == BOUNDS
    wildcat.attend(Q, res["Ks"], res["W"], rank, w.n_k, ws=ws)
    assert wildcat.check_device_status(ws) == BOUNDS
    # the context is intact: a valid pass still matches the first one
    again = wildcat.forward(Q, K, V, w.r, seed=1, ws=ws)
    assert wildcat.check_device_status(ws) == 0
    assert torch.equal(again["out"], res["out"])
