"""Builds libwildcat.so (sm_100a) in the package directory with nvcc, and its
bounds-checked twin libwildcat_debug.so (the same sources with
-DWC_DEBUG_BOUNDS=1: every data-dependent index is checked against its buffer
and a bad one is recorded as WC_ERR_BOUNDS instead of accessed).

    python -m coreset_attention_approximation_b200.build [--debug]
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libwildcat.so")
OBJDIR = os.path.join(HERE, "_build")
SOURCES = ["api.cu", "select.cu", "weights.cu", "expmm_simt.cu", "expmm_tc.cu", "attend.cu", "noalloc.cu",
           "center.cu", "stream_probe.cu"]
HEADERS = ["wc_common.cuh", "wc_internal.h", "wc_expmm.cuh", "wc_tc.cuh", "wc_exp2.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
]


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, jobs: int | None = None, debug: bool = False) -> str:
    objdir = OBJDIR + ("_debug" if debug else "")
    lib = os.path.join(HERE, "libwildcat_debug.so") if debug else LIB
    flags = FLAGS + (["-DWC_DEBUG_BOUNDS=1"] if debug else [])
    os.makedirs(objdir, exist_ok=True)
    include = os.path.join(os.path.dirname(HERE), "include", "wildcat.h")
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [include, __file__]
    objs, procs = [], []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        objs.append(obj)
        if _stale(obj, [path] + hdrs):
            cmd = [NVCC, *flags, "-c", path, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out.strip():
            print(out, file=sys.stderr)
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    if _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp,
                        "-lcudart", "-ldl"], check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(verbose=True, debug="--debug" in sys.argv[1:]))
