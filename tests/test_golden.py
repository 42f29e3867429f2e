"""The oracle still reproduces its stored values on the seeded tiny workload
(tests/golden/tiny_oracle.json, written by tests/golden/make_golden.py from
the oracle alone; the pages print no worked example)."""

import json
import os

import numpy as np

import oracle
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")


def test_oracle_reproduces_golden_tiny():
    g = json.load(open(GOLDEN))
    w = WORKLOADS[g["workload"]]
    Q, K, V = make_inputs(w, seed=g["seed"])
    res = oracle.forward(Q, K, V, w.r, seed=g["seed"])
    assert int(res["rank"][0, 0]) == g["rank"]
    assert res["piv"][0, 0].tolist() == g["piv"]
    assert np.allclose(res["W"][0, 0, 0], g["W_row0"], rtol=1e-12, atol=0)
    assert np.allclose(res["out"][0, 0, g["out_rows"]], g["out"], rtol=1e-12, atol=1e-15)
