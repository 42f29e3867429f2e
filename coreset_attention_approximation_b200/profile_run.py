"""Runs one stage of the path on a chosen workload, for profiler captures.

    python -m coreset_attention_approximation_b200.profile_run --workload kv --r 256 --stage select

Stages: select, weights, attend, forward.  Inputs are generated and copied to
the device first; the stage then runs `--reps` times (after `--warmup` runs)
and the device status is checked.  Prints the CUDA-event time per run.
"""

from __future__ import annotations

import argparse
import sys

import torch

from coreset_attention_approximation_b200 import wildcat
from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="kv", choices=sorted(WORKLOADS))
    ap.add_argument("--stage", default="select", choices=["select", "weights", "attend", "forward"])
    ap.add_argument("--r", type=int, default=None)
    ap.add_argument("--n", type=int, default=None)
    ap.add_argument("--heads", type=int, default=None, help="kv heads (query heads scale with them)")
    ap.add_argument("--reps", type=int, default=1)
    ap.add_argument("--warmup", type=int, default=0)
    args = ap.parse_args(argv)

    w = WORKLOADS[args.workload]
    over = {}
    if args.r:
        over["r"] = args.r
    if args.n:
        over["n_k"] = args.n
        if w.n_q == w.n_k:
            over["n_q"] = args.n
    if args.heads:
        over["hq"] = args.heads * (w.hq // w.hkv)
        over["hkv"] = args.heads
    w = w.replace(**over)
    dev = torch.device("cuda")
    Q, K, V = [t.to(dev) for t in make_inputs(w)]
    res = wildcat.forward(Q, K, V, w.r, seed=0)
    ws = res["ws"]

    def run():
        if args.stage == "select":
            wildcat.select(K, w.r, seed=0, ws=ws)
        elif args.stage == "weights":
            wildcat.weights(K, V, res["piv"], res["F"], res["rank"], w.r, ws=ws)
        elif args.stage == "attend":
            wildcat.attend(Q, res["Ks"], res["W"], res["rank"], w.n_k, ws=ws)
        else:
            wildcat.forward(Q, K, V, w.r, seed=0, ws=ws)

    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    for _ in range(args.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        print(f"{args.stage} {w.name} r={w.r} n={w.n_k} units={w.batch * w.hkv}: {e0.elapsed_time(e1):.3f} ms")
    status = wildcat.check_device_status(ws)
    if status != 0:
        print("device status:", wildcat.STATUS.get(status, status), file=sys.stderr)
        return 1
    return 0


if __name__ == "__main__":
    sys.exit(main())
