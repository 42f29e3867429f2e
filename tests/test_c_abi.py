"""The boundary is a C ABI: a plain C program (gcc, no C++, no torch) compiles
against include/wildcat.h, links libwildcat.so and calls the entry points that
need no GPU (sizes, status strings, argument checks)."""

import os
import subprocess

from coreset_attention_approximation_b200 import wildcat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "wildcat.h"

int main(void) {
    wc_shape s;
    memset(&s, 0, sizeof(s));
    s.batch = 1; s.hq = 8; s.hkv = 8; s.n_k = 131072; s.n_q = 131072;
    s.d = 128; s.dv = 128; s.r = 2048; s.dtype = WC_BF16; s.seed = 0; s.bins = 1;
    size_t ws = wc_workspace_bytes(&s), fws = wc_forward_workspace_bytes(&s);
    if (ws == 0 || fws <= ws || ws % 256) return 1;
    if (wc_f_ld(131072) != 131072 || wc_f_ld(65) != 128) return 2;
    if (strcmp(wc_status_string(WC_ERR_WORKSPACE), "workspace too small") != 0) return 3;
    wc_shape bad = s;
    bad.r = 0;
    if (wc_workspace_bytes(&bad) != 0) return 4;
    if (wc_select(&bad, (void*)256, (int32_t*)256, (float*)256, (int32_t*)256, (void*)256, ws, NULL) != WC_ERR_INVALID)
        return 5;
    if (wc_forward(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) != WC_ERR_INVALID) return 6;
    printf("%zu %zu\n", ws, fws);
    return 0;
}
"""


def test_plain_c_program_uses_the_library(tmp_path):
    lib = wildcat.LIB_PATH
    if not os.path.exists(lib):
        from coreset_attention_approximation_b200 import build

        build.build()
    src = tmp_path / "use_wildcat.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_wildcat"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe), "-L", libdir, "-lwildcat", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stderr)
    ws, fws = map(int, out.stdout.split())
    shape = wildcat.make_shape(1, 8, 8, 131072, 131072, 128, 128, 2048, wildcat.WC_BF16)
    assert ws == wildcat.workspace_bytes(shape) and fws == wildcat.forward_workspace_bytes(shape)
