"""bench.py on the CPU: the reference arm's JSON line (the oracle timed on the
host) and the algorithmic byte and flop counts the roofline divides by."""

import json
import os
import subprocess
import sys

import bench
from coreset_attention_approximation_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_counts_of_the_long_workload():
    w = WORKLOADS["long"]
    # per unit and step j: K read (n d 2), factor prefix read (4 n j), column written (4 n)
    n, r, d = w.n_k, w.r, w.d
    per_unit = sum(n * d * 2 + 4 * n * j + 4 * n for j in range(r))
    assert bench.select_bytes(w) == per_unit * w.hkv == 9350143803392
    f1, f2 = bench.gemm_flops(w)
    assert f1 == f2 == 2 * r * n * (d + w.dv + 1) * w.hkv
    # bins: each of B bins selects r / B pivots over n / B keys
    assert bench.select_bytes(w, bins=8) == 8 * w.hkv * sum((n // 8) * d * 2 + 4 * (n // 8) * (j + 1)
                                                            for j in range(r // 8))
    # centred keys stream as fp32
    assert bench.select_bytes(w, center=True) - bench.select_bytes(w) == n * r * d * 2 * w.hkv


def test_select_traffic_applies_only_to_the_captured_kernel_and_units():
    long_units = WORKLOADS["long"].hkv * WORKLOADS["long"].batch
    t = bench.select_traffic("long", "rpcholesky_kernel", long_units, 1, False)
    assert abs(t / bench.select_bytes(WORKLOADS["long"]) - 0.977058) < 1e-9
    # the long capture carries over to other unit counts (a strong split)
    assert bench.select_traffic("long", "rpcholesky_kernel", 1, 1, False) == t / long_units
    # another kernel, another unit count for a whole-workload capture, bins or centring: none
    assert bench.select_traffic("long", "rpcholesky_cluster_kernel", long_units, 1, False) is None
    assert bench.select_traffic("vit", "rpcholesky_unit_kernel", 768, 1, False) == 149619200 + 145093376
    assert bench.select_traffic("vit", "rpcholesky_unit_kernel", 96, 1, False) is None
    assert bench.select_traffic("vit", "rpcholesky_unit_kernel", 768, 4, False) is None
    assert bench.select_traffic("tiny", "rpcholesky_resident_kernel", 1, 1, True) is None
    assert bench.select_traffic("kv", "rpcholesky_kernel", 8, 1, False) is None
    assert bench.select_traffic("diffusion", "rpcholesky_kernel", 32, 1, False) is None
    assert bench.select_traffic("diffusion", "rpcholesky_cluster_kernel", 32, 1, False) == 9135514000 + 109580544


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "3", "--ref-pivots", "32"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["config"]["workload"] == "tiny" and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_approximation_error_of_exact_attention_is_zero():
    """The bench's accuracy report measures against exact softmax attention:
    handed the oracle's exact attention it reports (almost) zero, handed the
    coreset attention of a small coreset a clearly positive error."""
    import numpy as np
    import torch

    import oracle
    from coreset_attention_approximation_b200.workloads import make_inputs

    w = WORKLOADS["tiny"].replace(n_k=256, n_q=64, r=8)
    Q, K, V = make_inputs(w, seed=3)
    beta = 1.0 / np.sqrt(w.d)
    exact = torch.from_numpy(oracle.exact_attention(Q[0, 0], K[0, 0], V[0, 0], beta))[None, None].float()
    rep = bench.approximation_error(Q, K, V, exact, w, 1)
    assert rep["queries_per_head"] == 64 and rep["heads"] == 1 and rep["rel_err_max"] < 1e-5
    approx = torch.from_numpy(oracle.forward(Q, K, V, w.r, seed=0)["out"]).float()
    assert bench.approximation_error(Q, K, V, approx, w, 1)["rel_err_max"] > 1e-3
