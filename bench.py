"""WildCat forward throughput on B200: tokens/s, select HBM GB/s, GEMM TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl ours|reference]

A step is one pass of the whole path (select -> weights -> attend) over the
workload through the C ABI, inputs resident in HBM.  Default workload `long`:
8 heads, n = n_q = 131072 keys/queries, d = dv = 128, coreset r = 2048, bf16.
The inputs (K, V, Q: 805 MB) and the factor F (8.6 GB) are far larger than the
126 MB L2, so no flush is needed between steps.

With N > 1 (torchrun, one process per GPU) the (batch, kv head) units of one
problem are split across the ranks, with no collective on the data path (the
units are independent); the step time is the max over ranks:
  --scaling weak    (default) the problem is N workloads stacked along the
                    batch: rank k owns batch block k, drawn with its own seed,
                    and passes unit_base = k * units so its units draw the
                    Philox streams they draw in one call over the whole stack
  --scaling strong  the workload's own units, contiguous blocks of
                    [k U / N, (k + 1) U / N) per rank (U = batch * kv heads)
`--gather` adds one all-gather of the outputs after the timed region (timed
apart).  `--impl reference` times the CPU oracle on one whole unit of the same
workload (rank 0 only).
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from coreset_attention_approximation_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "WildCat forward tokens/sec at 1 B200; select HBM GB/s and GEMM TC-util vs peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of the select kernel per unit and launch on the named
# workload, from ncu's dram__bytes_read.sum + dram__bytes_write.sum (one-pass
# metrics) of the current select kernels:
#   long: the same 8 units and keys with r = 512 (670.081566 GB + 2.396902 GB
#     against 688.268509 GB of algorithmic bytes: 0.977058), applied to the
#     algorithmic bytes at r = 2048;
#   vit: the whole workload (149.6192 MB + 145.093376 MB over 768 units; the
#     keys are read once and the factor stays in L2);
#   tiny: the whole workload (193,536 bytes read, none written: the factor
#     stays in shared memory until it is written out);
#   diffusion: the whole workload (9.135514 GB + 109.580544 MB over 32 units:
#     keys and much of the factor stay in L2).
# Other workloads: not captured.
# Each entry: (the select kernel captured, units per launch then or None where
# the per-unit figure carries over to other unit counts, bytes per unit).
SELECT_DRAM_CAPTURES = {
    "long": ("rpcholesky_kernel", None, 0.977058 * 9350143803392 / 8),
    "vit": ("rpcholesky_unit_kernel", 768, (149619200 + 145093376) / 768),
    "tiny": ("rpcholesky_resident_kernel", 1, 193536.0),
    "diffusion": ("rpcholesky_cluster_kernel", 32, (9135514000 + 109580544) / 32),
}


def select_traffic(name, kernel, units, bins, center):
    """DRAM bytes of one select launch from the capture above, or None where
    none applies (another kernel, unit count, bins or centring)."""
    cap = SELECT_DRAM_CAPTURES.get(name)
    if cap is None or bins != 1 or center or cap[0] != kernel or (cap[1] is not None and cap[1] != units):
        return None
    return cap[2] * units


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def read_stream_gbs(dev, stream, gib: int = 4, reps: int = 5) -> float:
    """Read-only bandwidth of this GPU: the library's read probe streaming a
    buffer far larger than L2 (outside the timed region).  The select reads
    about five hundred bytes per byte it writes, so this figure, beside the
    copy bandwidth of MEASURED_PEAKS.json, is the other bound on it."""
    from coreset_attention_approximation_b200 import wildcat
    buf = torch.empty(gib << 30, dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(2):
        wildcat.read_probe(buf, sink, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        wildcat.read_probe(buf, sink, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = buf.numel()
    del buf
    return nbytes / (ms * 1e-3) / 1e9


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
    """Seed of batch block `rank` of the weak-scaling problem (block 0: `seed`)."""
    return seed + 1000003 * rank


def unit_range(units: int, world: int, rank: int) -> tuple[int, int]:
    """Rank `rank`'s contiguous block of `units` units: [rank U / N, (rank + 1) U / N)."""
    return rank * units // world, (rank + 1) * units // world


def local_problem(w, seed: int, world: int, rank: int, scaling: str):
    """This rank's share of the job: (Q, K, V host tensors, the workload those
    tensors form, unit_base, query tokens of the whole job per step).

    weak: the job is `world` copies of the workload stacked along the batch;
    rank k holds copy k (seed shard_seed(seed, k)), whose units are units
    k U .. (k + 1) U - 1 of the stack.  strong: the workload itself; rank k
    holds units unit_range(U, world, k), each unit as a batch entry of one kv
    head with its hq / hkv query heads."""
    U = w.batch * w.hkv
    if scaling == "weak" or world == 1:
        Q, K, V = make_inputs(w, seed=shard_seed(seed, rank))
        return Q, K, V, w, rank * U, world * w.batch * w.n_q
    lo, hi = unit_range(U, world, rank)
    if hi <= lo:
        raise SystemExit(f"--scaling strong needs at least one unit per rank ({U} units, {world} ranks)")
    group = w.hq // w.hkv
    Q, K, V = make_inputs(w, seed=seed)
    Qr = Q.reshape(U, group, w.n_q, w.d)[lo:hi].contiguous()
    Kr = K.reshape(U, 1, w.n_k, w.d)[lo:hi].contiguous()
    Vr = V.reshape(U, 1, w.n_k, w.dv)[lo:hi].contiguous()
    return Qr, Kr, Vr, w.replace(batch=hi - lo, hq=group, hkv=1), lo, w.batch * w.n_q


def gather_units(out_local, units: int, world: int, rank: int):
    """The strong split's outputs ([units_k, hq / hkv, n_q, dv] per rank, rank
    k holding unit_range(units, world, k)) assembled in unit order on every
    rank with one all-gather of equal-size blocks (padded to the largest
    share)."""
    import torch.distributed as dist

    per = max(unit_range(units, world, k)[1] - unit_range(units, world, k)[0] for k in range(world))
    lo, hi = unit_range(units, world, rank)
    buf = torch.zeros((per,) + tuple(out_local.shape[1:]), dtype=out_local.dtype, device=out_local.device)
    buf[: hi - lo] = out_local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    return torch.cat([parts[k][: unit_range(units, world, k)[1] - unit_range(units, world, k)[0]]
                      for k in range(world)])


def l2_note(w) -> str:
    """Whether a step's working set (Q, K, V, the factor F and the output)
    exceeds the 126 MB L2, so no flush is needed between steps."""
    es = 2 if w.dtype == "bf16" else 4
    units = w.batch * w.hkv
    ldf = (w.n_k + 63) // 64 * 64
    ws = (units * w.n_k * (w.d + w.dv) * es + w.batch * w.hq * w.n_q * (w.d * es + w.dv * 4)
          + units * w.r * ldf * 4)
    if ws > 126e6:
        return f"working set {ws / 1e6:.0f} MB > 126 MB L2 (no flush)"
    return f"working set {ws / 1e6:.0f} MB fits in the 126 MB L2 (no flush; L2-resident figures are context)"


def job_config(w, args, world: int) -> dict:
    """The `config` object of the JSON line, the same in both arms."""
    return {
        "workload": w.name, "batch": w.batch, "heads_q": w.hq, "heads_kv": w.hkv, "n_k": w.n_k,
        "n_q": w.n_q, "d": w.d, "dv": w.dv, "r": w.r, "keys": w.keys, "seed": args.seed,
        "bins": args.bins, "center": bool(args.center),
        "l2": l2_note(w),
        "parallelism": (f"{args.scaling} split of (batch, kv head) units over {world} ranks" if world > 1
                        else "one GPU, all units"),
    }


# ------------------------------------------------------------------ oracle on one unit

def oracle_unit(w, nq_s: int = 4096, bins: int = 1, center: bool = False, r_s: int | None = None):
    """Time the CPU oracle on one whole (batch, kv head) unit of workload `w`:
    unit 0's selection (every pivot step; with bins, every bin), its Nystrom
    weights, and attention for min(nq_s, n_q) queries of one of its query heads
    over its coreset (the union of the bins' coresets).  The workload's time is
    units x (select + weights) + query heads x attention x n_q / sampled
    queries: one multiplication by the unit count, and, when n_q > nq_s, the
    attention scaled by the query count (it is linear in the queries).
    r_s (tests only) cuts the selection to its first r_s steps per bin."""
    import oracle

    Q, K, V = make_inputs(w.replace(batch=1, hq=w.hq // w.hkv, hkv=1))
    beta = 1.0 / math.sqrt(w.d)
    nb, rb = w.n_k // bins, w.r // bins
    steps = rb if r_s is None else min(r_s, rb)
    nq_s = min(nq_s, w.n_q)
    Kn, Vn = K[0, 0].double().numpy(), V[0, 0].double().numpy()
    if center:
        Kn = oracle.center_keys(Kn)
    t_sel = t_w = 0.0
    Ks_parts, W_parts = [], []
    for b in range(bins):
        Kb, Vb = Kn[b * nb:(b + 1) * nb], Vn[b * nb:(b + 1) * nb]
        t0 = time.perf_counter()
        sel = oracle.rpcholesky(Kb, steps, beta, seed=0, unit=b)
        t1 = time.perf_counter()
        k = sel["rank"]
        if k > 0:
            W_parts.append(oracle.nystrom_weights(Kb, Vb, sel["piv"], k, beta))
            Ks_parts.append(Kb[sel["piv"][:k]])
        t2 = time.perf_counter()
        t_sel += t1 - t0
        t_w += t2 - t1
    t2 = time.perf_counter()
    oracle.coreset_attend(Q[0, 0, :nq_s].double().numpy(), np.concatenate(Ks_parts), np.concatenate(W_parts), beta)
    t_att = time.perf_counter() - t2
    units = w.batch * w.hkv
    heads = w.batch * w.hq
    total = units * (t_sel + t_w) + heads * t_att * (w.n_q / nq_s)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cut = f" (selection cut to {steps} of {rb} steps per bin: not a timing of the workload)" if steps < rb else ""
    return {
        "value": w.batch * w.n_q / total,
        "unit": "tokens/s",
        "cores": cores,
        "kind": "oracle",
        "sample": (f"{w.name}{f' bins={bins}' if bins > 1 else ''}{' centred' if center else ''}: unit 0 in full "
                   f"(select {t_sel:.1f} s, weights {t_w:.1f} s, attention {t_att:.2f} s for {nq_s} of {w.n_q} "
                   f"queries of one head), x {units} units and x {heads} heads x {w.n_q}/{nq_s} for attention: "
                   f"{total:.0f} s for the workload{cut}"),
        "sample_seconds": t_sel + t_w + t_att,
        "workload_seconds": total,
    }


# ------------------------------------------------------------------ GPU arm

def run_ours(args, world, rank, local):
    from coreset_attention_approximation_b200 import wildcat

    wj = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    # this rank's units (w: the workload they form on this GPU)
    Qh, Kh, Vh, w, unit_base, job_tokens = local_problem(wj, args.seed, world, rank, args.scaling)
    Q, K, V = Qh.to(dev), Kh.to(dev), Vh.to(dev)
    shape = wildcat.shape_of(Q, K, V, w.r, seed=args.seed, bins=args.bins, center=args.center, unit_base=unit_base)
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
                                bins=args.bins, center=args.center, unit_base=unit_base)

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
    sel_kernel = kernels.pop("select_kernel", "rpcholesky_kernel")
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
    alone.pop("select_kernel", None)

    peaks, which = load_peaks()
    read_gbs = read_stream_gbs(dev, stream)
    sel_avg = sum(sel_ms) / len(sel_ms)
    sb = select_bytes(w, args.bins, args.center)
    achieved = sb / (sel_avg * 1e-3) / 1e9
    f1, f2 = gemm_flops(w, args.bins)
    wts_avg, att_avg = sum(wts_ms) / len(wts_ms), sum(att_ms) / len(att_ms)
    traffic = select_traffic(w.name, sel_kernel, w.batch * w.hkv, args.bins, args.center)
    tokens = job_tokens
    gather = None
    if args.gather and world > 1 and args.scaling == "strong":
        # outputs of all ranks assembled in unit order on every rank (after the timed region)
        barrier(world)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        full = gather_units(out.reshape(w.batch, w.hq, w.n_q, w.dv), wj.batch * wj.hkv, world, rank)
        g1.record(stream)
        torch.cuda.synchronize()
        gather = {"ms": max_over_ranks(g0.elapsed_time(g1), world), "bytes_out": full.numel() * full.element_size(),
                  "collective": "all_gather (NCCL)"}
    res = {
        "metric": METRIC,
        "value": tokens / (ms_step * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": args.scaling,
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded generator; no dataset)",
        "config": job_config(wj, args, world),
        "roofline": {
            "bound": "hbm", "kernel": sel_kernel + " (select)", "achieved": achieved,
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "traffic": traffic, "peak_source": which,
            # the read-only stream this GPU reaches (the library's read probe), beside the copy peak
            "peak_read_gbs": read_gbs, "frac_read": achieved / read_gbs,
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
        "units_on_rank0": w.batch * w.hkv,
    }
    if gather:
        res["gather"] = gather
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
        m = re.search(r"expmm_(tc|simt|pair)_kernel<[^>]*?(\d)>", name)
        if m:
            # modes 0, 2: the weights' partial sums; 1: attention; 3: attention over a key split
            short = "attend_gemm" if m.group(2) in ("1", "3") else "weights_gemm"
        else:
            sk = re.search(r"rpcholesky_\w*kernel", name)
            if sk:
                # the streaming kernel, or a shared-memory form for short units
                out["select_kernel"] = sk.group(0)
            for key, tag in (("rpcholesky", "select"), ("gather_kernel", "gather"), ("to_half", "v_to_fp16"),
                             ("merge_c1", "merge_c1"), ("trsm_", "solve"),
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
    """The oracle as the reference arm: every timed step times one whole unit
    of the workload (oracle_unit) and scales it by the unit count.  A whole
    unit of the long workload takes about 40 s on 16 host cores, so the timed
    steps stop once `--ref-budget-s` seconds are spent (at least one runs);
    the warm-up steps run the selection's first pivots only."""
    w = WORKLOADS[args.workload]
    if rank != 0:
        return None
    for _ in range(args.warmup):
        oracle_unit(w, nq_s=256, bins=args.bins, center=args.center, r_s=min(16, w.r // args.bins))
    vals, last, spent = [], None, 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        last = oracle_unit(w, bins=args.bins, center=args.center, r_s=args.ref_pivots)
        vals.append(last["value"])
        dt = time.perf_counter() - t0
        spent += dt
        if spent + dt > args.ref_budget_s:   # the next whole unit would overrun the budget
            break
    v = statistics.median(vals)
    return {
        "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world, "steps": len(vals),
        "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": w.batch * w.n_q / v * 1e3,
        "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded generator; no dataset)",
        "config": job_config(w, args, world),
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
    ap.add_argument("--ref-pivots", type=int, default=None,
                    help="(tests only) cut the oracle's selection to this many steps per bin")
    ap.add_argument("--ref-budget-s", type=float, default=150.0,
                    help="reference arm: stop timing whole units once this many seconds are spent")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="N > 1: weak = N stacked workloads, one per rank; strong = the workload's units split")
    ap.add_argument("--gather", action="store_true",
                    help="strong scaling: all-gather the outputs after the timed region (timed apart)")
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
                cb = oracle_unit(WORKLOADS[args.workload], r_s=args.ref_pivots, bins=args.bins,
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
