"""A C program (no Python, no torch) runs the whole path through the C ABI on
the GPU: cudaMalloc'd buffers, wc_forward, wc_check_device_status.  Its inputs
and outputs go to files; the same inputs through the Python binding give the
same outputs bit for bit."""

import os
import subprocess

import numpy as np
import pytest
import torch

from coreset_attention_approximation_b200 import wildcat

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime.h>
#include "wildcat.h"

/* bf16 bits of a value in [-2, 2) drawn from a 64-bit LCG */
static uint16_t next_bf16(uint64_t* st) {
    *st = *st * 6364136223846793005ull + 1442695040888963407ull;
    float f = ((float)(*st >> 40) / 16777216.0f) * 4.0f - 2.0f;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static int put(const char* path, const void* p, size_t n) {
    FILE* f = fopen(path, "wb");
    if (!f) return 1;
    size_t w = fwrite(p, 1, n, f);
    fclose(f);
    return w != n;
}

int main(int argc, char** argv) {
    if (argc < 2) return 90;
    const char* dir = argv[1];
    wc_shape s;
    memset(&s, 0, sizeof(s));
    s.batch = 1; s.hq = 4; s.hkv = 2; s.n_k = 3000; s.n_q = 700; s.d = 64; s.dv = 64; s.r = 200;
    s.dtype = WC_BF16; s.seed = 9; s.bins = 1;
    const size_t nq = (size_t)s.batch * s.hq * s.n_q * s.d, nk = (size_t)s.batch * s.hkv * s.n_k * s.d;
    const size_t nv = (size_t)s.batch * s.hkv * s.n_k * s.dv, no = (size_t)s.batch * s.hq * s.n_q * s.dv;
    uint16_t* hq = malloc(nq * 2);
    uint16_t* hk = malloc(nk * 2);
    uint16_t* hv = malloc(nv * 2);
    float* ho = malloc(no * 4);
    uint64_t st = 12345;
    for (size_t i = 0; i < nq; ++i) hq[i] = next_bf16(&st);
    for (size_t i = 0; i < nk; ++i) hk[i] = next_bf16(&st);
    for (size_t i = 0; i < nv; ++i) hv[i] = next_bf16(&st);
    void *dq, *dk, *dv, *dws;
    float* dout;
    const size_t ws = wc_forward_workspace_bytes(&s);
    if (ws == 0) return 91;
    if (cudaMalloc(&dq, nq * 2) || cudaMalloc(&dk, nk * 2) || cudaMalloc(&dv, nv * 2) ||
        cudaMalloc((void**)&dout, no * 4) || cudaMalloc(&dws, ws))
        return 92;
    cudaMemset(dws, 0, ws);
    cudaMemcpy(dq, hq, nq * 2, cudaMemcpyHostToDevice);
    cudaMemcpy(dk, hk, nk * 2, cudaMemcpyHostToDevice);
    cudaMemcpy(dv, hv, nv * 2, cudaMemcpyHostToDevice);
    wc_status e = wc_forward(&s, dq, dk, dv, dout, NULL, NULL, NULL, NULL, NULL, dws, ws, NULL);
    if (e != WC_OK) { fprintf(stderr, "%s\n", wc_status_string(e)); return 93; }
    e = wc_check_device_status(dws, NULL);
    if (e != WC_OK) { fprintf(stderr, "%s\n", wc_status_string(e)); return 94; }
    cudaMemcpy(ho, dout, no * 4, cudaMemcpyDeviceToHost);
    char path[4096];
    snprintf(path, sizeof(path), "%s/q.bin", dir); if (put(path, hq, nq * 2)) return 95;
    snprintf(path, sizeof(path), "%s/k.bin", dir); if (put(path, hk, nk * 2)) return 95;
    snprintf(path, sizeof(path), "%s/v.bin", dir); if (put(path, hv, nv * 2)) return 95;
    snprintf(path, sizeof(path), "%s/out.bin", dir); if (put(path, ho, no * 4)) return 95;
    cudaFree(dq); cudaFree(dk); cudaFree(dv); cudaFree(dout); cudaFree(dws);
    free(hq); free(hk); free(hv); free(ho);
    return 0;
}
"""


def _bf16(path, shape):
    raw = np.fromfile(path, dtype=np.int16)          # the bf16 bit patterns
    return torch.from_numpy(raw).view(torch.bfloat16).reshape(shape)


def test_c_program_runs_the_path_through_the_abi(tmp_path):
    lib = wildcat.LIB_PATH
    libdir = os.path.dirname(lib)
    src = tmp_path / "forward.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "forward"
    cuda = "/usr/local/cuda"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-I", os.path.join(ROOT, "include"), "-I", f"{cuda}/include",
                    str(src), "-o", str(exe), "-L", libdir, "-lwildcat", f"-Wl,-rpath,{libdir}",
                    "-L", f"{cuda}/lib64", "-lcudart", f"-Wl,-rpath,{cuda}/lib64"], check=True)
    run = subprocess.run([str(exe), str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, (run.returncode, run.stderr)
    Q = _bf16(tmp_path / "q.bin", (1, 4, 700, 64))
    K = _bf16(tmp_path / "k.bin", (1, 2, 3000, 64))
    V = _bf16(tmp_path / "v.bin", (1, 2, 3000, 64))
    out_c = torch.from_numpy(np.fromfile(tmp_path / "out.bin", dtype=np.float32).reshape(1, 4, 700, 64))
    res = wildcat.forward(Q.cuda(), K.cuda(), V.cuda(), 200, seed=9)
    torch.cuda.synchronize()
    assert torch.isfinite(out_c).all()
    assert torch.equal(res["out"].cpu(), out_c)
