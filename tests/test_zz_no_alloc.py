"""wc_attend_noalloc — attention for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or pass a workspace (an allocator that must
not be re-entered, a memory budget fixed before the first call, a plugin that
only receives its tensors).  For them the library keeps the attention step's
scratch in a fixed device array of its own.  These tests call that entry point
through the C ABI twice in a row, on two different shapes (the array is
shared and keeps the previous call's contents), and check each output
against wc_attend, which runs the same step with a caller workspace, within
the tolerance the parity tests use; one shape with key bins is also checked
against the oracle.  They check that warm calls change neither torch's
allocations nor the device's free memory, and that a shape needing more than
the array holds is refused before any launch.

The file is named to run last: a run that stops at the first failure has then
already run every other test.
"""

import numpy as np
import pytest
import torch

import oracle
from coreset_attention_approximation_b200 import wildcat
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs
from parity import TOL_OUT, rel_err

pytestmark = pytest.mark.gpu


def _coreset(w, seed, **kw):
    Q, K, V = [t.cuda() for t in make_inputs(w, seed=seed)]
    res = wildcat.forward(Q, K, V, w.r, seed=seed, **kw)
    torch.cuda.synchronize()
    # the forward pass that built the coreset ran clean
    assert wildcat.check_device_status(res["ws"]) == 0
    return Q, res


@pytest.mark.parametrize("order", [0, 1])
def test_noalloc_attend_matches_workspace_attend_twice(order):
    shapes = [WORKLOADS["diffusion"].replace(batch=1, hq=4, hkv=4, n_k=2048, n_q=700),
              WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=4096, r=300, n_q=129)]
    if order:
        shapes = shapes[::-1]
    for k, w in enumerate(shapes):
        Q, res = _coreset(w, seed=10 + k)
        want = wildcat.attend(Q, res["Ks"], res["W"], res["rank"], w.n_k)
        got = wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k)
        torch.cuda.synchronize()
        for b in range(w.batch):
            for h in range(w.hq):
                assert rel_err(got[b, h].cpu().numpy(), want[b, h].cpu().numpy()) <= TOL_OUT[torch.bfloat16]


def test_noalloc_attend_with_bins_matches_the_oracle():
    # 4 bins: attention over the union of the bins' coresets (all r rows count)
    w = WORKLOADS["diffusion"].replace(batch=1, hq=2, hkv=2, n_k=2048, n_q=333, r=128)
    Qh, Kh, Vh = make_inputs(w, seed=21)
    Q, res = _coreset(w, seed=21, bins=4)
    got = wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k, bins=4)
    again = wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k, bins=4)
    want = wildcat.attend(Q, res["Ks"], res["W"], res["rank"], w.n_k, bins=4)
    torch.cuda.synchronize()
    assert torch.equal(got, again)          # a second call over the left-behind scratch
    piv = res["piv"].cpu().numpy()
    rank3 = res["rank"].cpu().numpy().reshape(w.batch, w.hkv, 4)
    o = oracle.forward(Qh, Kh, Vh, w.r, seed=21, replay=(piv, rank3), bins=4)
    for h in range(w.hq):
        assert rel_err(got[0, h].cpu().numpy(), want[0, h].cpu().numpy()) <= TOL_OUT[torch.bfloat16]
        assert rel_err(got[0, h].cpu().numpy(), o["out"][0, h]) <= TOL_OUT[torch.bfloat16]


def test_noalloc_attend_fp32_runs_without_scratch():
    w = WORKLOADS["tiny"]
    Qh, Kh, Vh = make_inputs(w, seed=0)
    Q, res = _coreset(w, seed=0)
    want = wildcat.attend(Q, res["Ks"], res["W"], res["rank"], w.n_k)
    got = wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k)
    torch.cuda.synchronize()
    assert rel_err(got[0, 0].cpu().numpy(), want[0, 0].cpu().numpy()) <= TOL_OUT[torch.float32]
    o = oracle.forward(Qh, Kh, Vh, w.r, seed=0, replay=(res["piv"].cpu().numpy(), res["rank"].cpu().numpy()))
    assert rel_err(got[0, 0].cpu().numpy(), o["out"][0, 0]) <= TOL_OUT[torch.float32]


def test_warm_noalloc_calls_allocate_nothing():
    w = WORKLOADS["kv"].replace(hq=8, hkv=2, n_k=4096, r=256, n_q=300)
    Q, res = _coreset(w, seed=5)
    out = torch.empty(w.batch, w.hq, w.n_q, w.dv, dtype=torch.float32, device="cuda")
    wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k, out=out)   # warm: code loaded
    torch.cuda.synchronize()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        wildcat.attend_noalloc(Q, res["Ks"], res["W"], res["rank"], w.n_k, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0 and torch.cuda.memory_reserved() == reserved0
    assert free1 == free0
    want = wildcat.attend(Q, res["Ks"], res["W"], res["rank"], w.n_k)
    for h in range(w.hq):
        assert rel_err(out[0, h].cpu().numpy(), want[0, h].cpu().numpy()) <= TOL_OUT[torch.bfloat16]


def test_noalloc_attend_refuses_shapes_beyond_its_scratch():
    # 64 kv heads x r = 2048 x dv = 128 needs 32 MiB of fp16 weights alone
    B, Hq, Hkv, r, d, dv, nq = 1, 64, 64, 2048, 128, 128, 128
    Q = torch.zeros(B, Hq, nq, d, dtype=torch.bfloat16, device="cuda")
    Ks = torch.zeros(B, Hkv, r, d, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(B, Hkv, r, dv + 1, dtype=torch.float32, device="cuda")
    rank = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    with pytest.raises(wildcat.WildcatError) as e:
        wildcat.attend_noalloc(Q, Ks, W, rank, 4096)
    assert e.value.code == 5
