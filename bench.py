"""WildCat forward throughput on B200: tokens/s, select HBM GB/s, GEMM TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl ours|reference]

A step is one pass of the whole path (select -> weights -> attend) over the
workload through the C ABI, inputs resident in HBM.  Default workload `long`:
8 heads, n = n_q = 131072 keys/queries, d = dv = 128, coreset r = 2048, bf16.
The inputs (K, V, Q: 805 MB) and the factor F (8.6 GB) are far larger than the
126 MB L2, so no flush is needed between steps.

With N > 1 (torchrun, one process per GPU) every rank runs its own copy of the
workload (independent units, no collective on the data path: weak scaling);
the step time is the max over ranks.  `--impl reference` times the CPU oracle
on a bounded sample of the same workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "WildCat forward tokens/sec at 1 B200; select HBM GB/s and GEMM TC-util vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# dram bytes (read + write) per select launch per unit, from a one-pass ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of the current select
# kernel on the named workload: long = 9.306759 TB + 8.881209 GB over 8 units
# (profiles/select_rpcholesky_long8.md).  Other workloads: not captured.
SELECT_DRAM_BYTES_PER_UNIT = {"long": (9.306759e12 + 8.881209e9) / 8}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def select_bytes(w, bins: int = 1, center: bool = False) -> float:
    """Algorithmic bytes of one select launch: per unit (per bin with bins) and
    pivot step j, one read of K (n d s_K), of the factor prefix F[:, :j] (4 n j)
    and one write of the new column (4 n).  Centred keys stream as fp32."""
    sk = 2 if (w.dtype == "bf16" and not center) else 4
    n, r, d = w.n_k // bins, w.r // bins, w.d
    per_unit = n * r * d * sk + 2.0 * n * r * (r - 1) + 4.0 * n * r
    return per_unit * w.batch * w.hkv * bins


def gemm_flops(w, bins: int = 1) -> tuple[float, float]:
    """Tensor-core contraction flops: C1 = exp(K_S K^T)[V|1] per unit (per bin:
    r/B coreset rows against n/B keys) and A = exp(Q K_S^T) W per query head
    over all r coreset rows, the [V|1] column counted."""
    f1 = 2.0 * w.r * w.n_k * (w.d + w.dv + 1) * w.batch * w.hkv / bins
    f2 = 2.0 * w.n_q * w.r * (w.d + w.dv + 1) * w.batch * w.hq
    return f1, f2


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def _lines(self):
        try:
            with open(self.file.name) as f:
                return sum(1 for line in f if line.strip())
        except OSError:
            return 0

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # the first sample lands before the timed region starts (nvidia-smi takes a moment to come up)
        t0 = time.time()
        while self.proc is not None and self._lines() == 0 and time.time() - t0 < 5.0:
            time.sleep(0.02)
        self.n_enter = self._lines()
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            # a short timed region still gets the sample that follows it
            t0 = time.time()
            while self._lines() <= self.n_enter and time.time() - t0 < 1.0:
                time.sleep(0.02)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self):
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for k, nm in enumerate(names):
                if len(r) > 5 + k and r[5 + k].strip() == "Active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ ranks

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(seed: int, rank: int) -> int:
    """Each rank draws its own independent copy of the workload."""
    return seed + 1000003 * rank


# ------------------------------------------------------------------ oracle sample

def oracle_sample(w, r_s: int = 512, nq_s: int = 4096, bins: int = 1, center: bool = False):
    """Time the CPU oracle on a bounded sample of workload `w` and scale it to
    the whole workload.  Sample: unit 0, select steps 0..r_s-1 (the select's
    cost is n * sum_j (d + j) multiply-adds, so its time scales by that count),
    the weights on those r_s pivots (C1 dominates: linear in r) and attention
    for nq_s queries of one head (linear in queries and in r).  With bins the
    select and weights sample is bin 0 of unit 0 (n/B keys, r/B pivots), scaled
    by units x B; attention still covers r coreset rows."""
    import numpy as np

    import oracle

    Q, K, V = make_inputs(w.replace(batch=1, hq=w.hq // w.hkv, hkv=1))
    beta = 1.0 / math.sqrt(w.d)
    nb, rb = w.n_k // bins, w.r // bins
    r_s = min(r_s, rb)
    nq_s = min(nq_s, w.n_q)
    Kn, Vn = K[0, 0].double().numpy(), V[0, 0].double().numpy()
    if center:
        Kn = oracle.center_keys(Kn)
    Kn, Vn = Kn[:nb], Vn[:nb]
    t0 = time.perf_counter()
    sel = oracle.rpcholesky(Kn, r_s, beta, seed=0, unit=0)
    t1 = time.perf_counter()
    k = sel["rank"]
    Wt = oracle.nystrom_weights(Kn, Vn, sel["piv"], k, beta)
    t2 = time.perf_counter()
    oracle.coreset_attend(Q[0, 0, :nq_s].double().numpy(), Kn[sel["piv"][:k]], Wt, beta)
    t3 = time.perf_counter()

    def sel_work(r):
        return nb * (r * w.d + r * (r - 1) / 2.0)

    units = w.batch * w.hkv * bins
    heads = w.batch * w.hq
    t_sel = (t1 - t0) * sel_work(rb) / sel_work(r_s)
    t_w = (t2 - t1) * rb / r_s
    t_att = (t3 - t2) * (w.n_q / nq_s) * (w.r / r_s)
    total = units * (t_sel + t_w) + heads * t_att
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {
        "value": w.batch * w.n_q / total,
        "unit": "tokens/s",
        "cores": cores,
        "kind": "oracle",
        "sample": (f"{w.name}{f' bins={bins}' if bins > 1 else ''}{' centred' if center else ''}: "
                   f"unit 0 of {units}; select steps 0..{r_s - 1} of {rb} "
                   f"({t1 - t0:.1f} s, scaled by n*sum_j(d+j)); weights on {r_s} pivots ({t2 - t1:.1f} s, "
                   f"scaled x r/{r_s}); attend {nq_s} queries ({t3 - t2:.1f} s, scaled x n_q/{nq_s} x r/{r_s}); "
                   f"whole-workload estimate {total:.0f} s"),
        "sample_seconds": t3 - t0,
    }


# ------------------------------------------------------------------ GPU arm

def run_ours(args, world, rank, local):
    from coreset_attention_approximation_b200 import wildcat

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    Qh, Kh, Vh = make_inputs(w, seed=shard_seed(args.seed, rank))
    Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
    shape = wildcat.shape_of(Q, K, V, w.r, seed=args.seed, bins=args.bins, center=args.center)
    ws = wildcat.workspace(shape, dev)
    o = wildcat._outputs(shape, dev, K.dtype)
    out = torch.empty(w.batch, w.hq, w.n_q, w.dv, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    lib = wildcat.lib()
    import ctypes

    sp = ctypes.byref(shape)
    P = wildcat._ptr
    st = wildcat._stream(stream)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        wildcat._check(lib.wc_select(sp, P(K), P(o["piv"]), P(o["F"]), P(o["rank"]), P(ws), ws.numel(), st),
                       "wc_select")
        if ev:
            ev[1].record(stream)
        wildcat._check(lib.wc_weights(sp, P(K), P(V), P(o["piv"]), P(o["F"]), P(o["rank"]), P(o["Ks"]),
                                      P(o["W"]), P(ws), ws.numel(), st), "wc_weights")
        if ev:
            ev[2].record(stream)
        wildcat._check(lib.wc_attend(sp, P(Q), P(o["Ks"]), P(o["W"]), P(o["rank"]), P(out), P(ws),
                                     ws.numel(), st), "wc_attend")
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = wildcat.check_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {wildcat.STATUS.get(status, status)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_begin.record(stream)
        for k in range(args.steps):
            step(evs[k])
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    status = wildcat.check_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after timed steps: {wildcat.STATUS.get(status, status)}")
    total_ms = t_begin.elapsed_time(t_end)
    sel_ms = [e[0].elapsed_time(e[1]) for e in evs]
    wts_ms = [e[1].elapsed_time(e[2]) for e in evs]
    att_ms = [e[2].elapsed_time(e[3]) for e in evs]
    ms_step = max_over_ranks(total_ms / args.steps, world)

    # ---- e2e: the same steps from pinned host buffers through the binding's
    # host pipeline: every step copies its Q, K, V in and its output back, the
    # copies of the neighbouring steps overlapping this step's compute
    Qp, Kp, Vp = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
    outp = [torch.empty(out.shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    h2d = Qp.numel() * Qp.element_size() + Kp.numel() * Kp.element_size() + Vp.numel() * Vp.element_size()
    d2h = outp[0].numel() * outp[0].element_size()
    pipe = wildcat.HostPipeline(Qp, Kp, Vp, w.r, seed=args.seed, device=dev, stream=stream, ws=ws, outputs=o,
                                bins=args.bins, center=args.center)

    def batches(k):
        return [(Qp, Kp, Vp, outp[i % 2]) for i in range(k)]

    pipe.run(batches(2))
    if pipe.wait() != 0:
        raise RuntimeError("device status after e2e warm-up")
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    pipe.run(batches(args.steps))
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    if pipe.wait() != 0:
        raise RuntimeError("device status after e2e steps")
    del pipe

    kernels = kernel_breakdown(step)
    approx = approximation_error(Q, K, V, out, w, args.bins)

    def gemm_steps():
        # weights and attention back to back, without the select before them
        for _ in range(4):
            wildcat._check(lib.wc_weights(sp, P(K), P(V), P(o["piv"]), P(o["F"]), P(o["rank"]), P(o["Ks"]),
                                          P(o["W"]), P(ws), ws.numel(), st), "wc_weights")
            wildcat._check(lib.wc_attend(sp, P(Q), P(o["Ks"]), P(o["W"]), P(o["rank"]), P(out), P(ws),
                                         ws.numel(), st), "wc_attend")

    alone = kernel_breakdown(gemm_steps)
    alone.pop("launches", None)

    peaks, which = load_peaks()
    sel_avg = sum(sel_ms) / len(sel_ms)
    sb = select_bytes(w, args.bins, args.center)
    achieved = sb / (sel_avg * 1e-3) / 1e9
    f1, f2 = gemm_flops(w, args.bins)
    wts_avg, att_avg = sum(wts_ms) / len(wts_ms), sum(att_ms) / len(att_ms)
    captured = w.name in SELECT_DRAM_BYTES_PER_UNIT and args.bins == 1 and not args.center
    traffic = SELECT_DRAM_BYTES_PER_UNIT[w.name] * w.batch * w.hkv if captured else None
    tokens = w.batch * w.n_q * world
    res = {
        "metric": METRIC,
        "value": tokens / (ms_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded generator; no dataset)",
        "config": {
            "workload": w.name, "batch": w.batch, "heads_q": w.hq, "heads_kv": w.hkv, "n_k": w.n_k,
            "n_q": w.n_q, "d": w.d, "dv": w.dv, "r": w.r, "keys": w.keys, "seed": args.seed,
            "bins": args.bins, "center": bool(args.center),
            "l2": "inputs and factor larger than L2 (no flush)",
            "parallelism": f"independent units per rank x{world}",
        },
        "roofline": {
            "bound": "hbm", "kernel": "rpcholesky_kernel (select)", "achieved": achieved,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "traffic": traffic, "peak_source": which,
            "algorithmic_bytes_per_launch": sb, "launch_ms": sel_avg,
        },
        "stages_ms": {"select": sel_avg, "weights": wts_avg, "attend": att_avg},
        # the KV-cache views: compress (select + weights) once, then attend
        "compress_ms": sel_avg + wts_avg,
        "attend_tokens_per_s": tokens / (att_avg * 1e-3),
        "compress_attend_tokens_per_s": tokens / ((sel_avg + wts_avg + att_avg) * 1e-3),
        "gemm": gemm_report(kernels, f1, f2, peaks),
        "gemm_alone": gemm_alone_report(alone, f1, f2, peaks),
        "approximation": approx,
        "kernels_ms": kernels,
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "copies": "double-buffered: step i+1 in and step i-1 out overlap step i"},
        # counted on the profiled step (the same launches as every timed step)
        "gpu_launches": kernels.pop("launches") * args.steps,
        "clocks": clocks.summary(),
    }
    return res


def kernel_breakdown(step):
    """Device time of each kernel of one extra step (outside the timed
    region), from CUPTI activity records via torch.profiler."""
    from torch.profiler import ProfilerActivity, profile

    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize()
    import re

    out = {"launches": 0}
    for ev in prof.events():
        if ev.device_type.name != "CUDA":
            continue
        name = ev.name
        if "wc::" in name:
            out["launches"] += 1          # this library's kernels (namespace wc)
        short = None
        m = re.search(r"expmm_(tc|simt)_kernel<[^>]*?(\d)>", name)
        if m:
            # modes 0, 2: the weights' partial sums; 1: attention; 3: attention over a key split
            short = "attend_gemm" if m.group(2) in ("1", "3") else "weights_gemm"
        else:
            for key, tag in (("rpcholesky", "select"), ("gather_kernel", "gather"), ("to_half", "v_to_fp16"),
                             ("merge_c1", "merge_c1"), ("trsm_kernel", "solve"),
                             ("weights_prep", "w_prep"), ("key_shift", "shift"),
                             ("attend_combine", "attend_combine")):
                if key in name:
                    short = tag
                    break
        if short:
            out[short] = out.get(short, 0.0) + ev.device_time / 1e3
    return out


def gemm_report(kernels, f1, f2, peaks):
    """Tensor-core utilisation of the two exp-GEMMs.  They run inside a
    seconds-long step right after the select, under the power cap, so `frac`
    is against the sustained bf16 figure (a GEMM loop held for seconds);
    `frac_burst` against the burst figure is shown beside it."""
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained") or burst
    rep = {"peak_tflops_bf16": burst, "peak_tflops_bf16_sustained": sustained, "frac_of": "sustained"}
    for name, flops in (("weights_gemm", f1), ("attend_gemm", f2)):
        ms = kernels.get(name)
        if ms:
            tf = flops / (ms * 1e-3) / 1e12
            rep[name] = {"ms": ms, "tflops": tf, "frac": tf / sustained, "frac_burst": tf / burst, "flops": flops}
    return rep


def approximation_error(Q, K, V, out, w, bins, nq_s=4096, max_heads=16):
    """How far the coreset attention is from exact softmax attention (for
    reporting only, outside the timed region): exact attention in fp32 with
    plain torch matmuls on a seeded subsample of at most `nq_s` queries per head
    (the first `max_heads` query heads), against the path's output rows.
    ||out - exact||_F / ||exact||_F per head, and the largest entrywise error
    over the largest |V| entry of the head."""
    beta = 1.0 / math.sqrt(w.d)
    g = torch.Generator().manual_seed(0)
    idx = torch.randperm(w.n_q, generator=g)[:min(nq_s, w.n_q)].to(Q.device)
    group = w.hq // w.hkv
    errs, ents = [], []
    with torch.no_grad():
        for z in range(min(w.batch * w.hq, max_heads)):
            b, h = divmod(z, w.hq)
            q = Q[b, h, idx].float()
            k, v = K[b, h // group].float(), V[b, h // group].float()
            exact = torch.cat([torch.softmax((q[i:i + 512] @ k.T) * beta, dim=-1) @ v
                               for i in range(0, q.shape[0], 512)])
            diff = out[b, h, idx] - exact
            errs.append(float(diff.norm() / exact.norm()))
            ents.append(float(diff.abs().max() / v.abs().max()))
    return {"kind": "against exact softmax attention in fp32 on sampled queries",
            "queries_per_head": int(idx.numel()), "heads": len(errs), "bins": bins,
            "rel_err_mean": statistics.mean(errs), "rel_err_max": max(errs),
            "max_abs_err_over_max_v": max(ents)}


def gemm_alone_report(kernels, f1, f2, peaks):
    """The two exp-GEMMs timed alone (four weights + attention passes back to
    back, no select between them; average per launch), against the burst bf16
    figure."""
    burst = peaks["bf16_tflops"]
    rep = {"peak_tflops_bf16": burst, "frac_of": "burst", "passes": 4}
    for name, flops in (("weights_gemm", f1), ("attend_gemm", f2)):
        ms = kernels.get(name)
        if ms:
            ms /= 4
            tf = flops / (ms * 1e-3) / 1e12
            rep[name] = {"ms": ms, "tflops": tf, "frac": tf / burst}
    return rep


def run_reference(args, world, rank):
    w = WORKLOADS[args.workload]
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_sample(w, r_s=64, nq_s=256, bins=args.bins, center=args.center)
    vals = []
    last = None
    for _ in range(args.steps):
        last = oracle_sample(w, r_s=args.ref_pivots, nq_s=4096, bins=args.bins, center=args.center)
        vals.append(last["value"])
    v = statistics.median(vals)
    return {
        "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": w.batch * w.n_q / v * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator; no dataset)",
        "config": {"workload": w.name, "batch": w.batch, "heads_q": w.hq, "heads_kv": w.hkv, "n_k": w.n_k,
                   "n_q": w.n_q, "d": w.d, "dv": w.dv, "r": w.r, "keys": w.keys, "seed": args.seed,
                   "bins": args.bins, "center": bool(args.center)},
        "impl": "reference",
        "cpu_baseline": {k: last[k] for k in ("value", "unit", "cores", "kind", "sample")} | {"value": v},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="long", choices=sorted(WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-pivots", type=int, default=512, help="select steps in the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bins", type=int, default=1,
                    help="divide-and-conquer selection: B key bins per head (n and r multiples of B)")
    ap.add_argument("--center", action="store_true", help="centre the keys before selection and weights")
    args = ap.parse_args()
    if args.warmup < 3:
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3

    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_ours(args, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                cb = oracle_sample(WORKLOADS[args.workload], r_s=args.ref_pivots, bins=args.bins,
                                   center=args.center)
                res["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
