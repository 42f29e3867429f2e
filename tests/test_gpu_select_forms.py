"""Each form of the select runs where the launcher sends it and matches the
oracle there: the resident cluster (one 512-key head), one block per unit (many
1024-key heads), a cluster per unit (32 heads of 4096 keys) and the streaming
kernel (two heads of 32768 keys).  Pivots identical, F within 1e-5 and outputs
within the dtype's tolerance of the fp64 oracle; the kernel that ran is read
from the profiler's launch records."""

import re

import pytest
import torch
from torch.profiler import ProfilerActivity, profile

from coreset_attention_approximation_b200 import wildcat
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs
from parity import compare

pytestmark = pytest.mark.gpu

CASES = [
    ("rpcholesky_resident_kernel", WORKLOADS["tiny"]),
    ("rpcholesky_unit_kernel", WORKLOADS["vit"].replace(batch=2, hq=80, hkv=80, n_q=128)),
    ("rpcholesky_cluster_kernel", WORKLOADS["diffusion"].replace(r=48, n_q=256)),
    ("rpcholesky_kernel", WORKLOADS["long"].replace(hq=2, hkv=2, n_k=32768, n_q=256, r=24)),
]


def select_kernel(K, r):
    Kd = K.cuda()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        wildcat.select(Kd, r, seed=0)
        torch.cuda.synchronize()
    names = {m.group(0) for e in prof.events() if e.device_type.name == "CUDA"
             for m in [re.search(r"rpcholesky_\w*kernel", e.name)] if m}
    return names


@pytest.mark.parametrize("kernel,w", CASES, ids=[c[0] for c in CASES])
def test_select_form_runs_and_matches_the_oracle(kernel, w):
    Q, K, V = make_inputs(w)
    assert select_kernel(K, w.r) == {kernel}
    compare(Q, K, V, w.r)
