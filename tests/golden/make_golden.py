"""Writes tests/golden/tiny_oracle.json from the oracle alone.

No page of the method prints a worked example (no pivot list, weight or
output value), so the stored values here are the oracle's own, on the seeded
`tiny` workload (1 head, n = 512, d = 64, r = 32, fp32, seed 0).  They guard
against an unannounced change of the oracle's arithmetic; what makes them
right is the pin suite in tests/test_oracle_*.py.

Run from the repository root:  python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs  # noqa: E402


def main():
    w = WORKLOADS["tiny"]
    Q, K, V = make_inputs(w, seed=0)
    res = oracle.forward(Q, K, V, w.r, seed=0)
    rows = [0, 1, 100, 255, 511]
    out = {
        "workload": "tiny", "seed": 0, "beta": res["beta"], "eps_stop": oracle.DEFAULT_EPS_STOP,
        "rank": int(res["rank"][0, 0]),
        "piv": res["piv"][0, 0].tolist(),
        "W_row0": res["W"][0, 0, 0].tolist(),
        "out_rows": rows,
        "out": res["out"][0, 0, rows].tolist(),
    }
    path = os.path.join(ROOT, "tests", "golden", "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
