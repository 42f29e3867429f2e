"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of wc_oracle.c (a dropped term, a
wrong sign, a transposed operand, an off-by-one comparison, a wrong constant),
builds it into a temporary library, and runs the oracle pin suite against it
in a child process (WC_ORACLE_LIB points the loader at the broken build).
The suite must fail for every mutant.
"""

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "wc_oracle.c")
PINS = ["tests/test_oracle_philox.py", "tests/test_oracle_select.py", "tests/test_oracle_weights_attend.py"]

MUTANTS = {
    "drop_correction": ("g -= Fi[c] * Fs[c];", "g -= 0.0 * Fi[c] * Fs[c];"),
    "correction_wrong_operand": ("g -= Fi[c] * Fs[c];", "g -= Fi[c] * Fi[c];"),
    "downdate_sign": ("const double nd = dg[i] - f * f;", "const double nd = dg[i] + f * f;"),
    "cdf_ge": ("if (found < 0 && run > t) found = i;", "if (found < 0 && run >= t) found = i;"),
    "keep_earlier_pivots": ("F[(size_t)piv[c] * r + j] = 0.0;", "(void)0;"),
    "philox_weyl": ("k[1] += 0xBB67AE85u;", "k[1] += 0xBB67AE84u;"),
    "philox_mix": ("const uint32_t y0 = (uint32_t)(p1 >> 32) ^ x[1] ^ k[0];",
                   "const uint32_t y0 = (uint32_t)(p1 >> 32) ^ x[3] ^ k[0];"),
    "uniform_word": ("return (double)out[0] * (1.0 / 4294967296.0);", "return (double)out[1] * (1.0 / 4294967296.0);"),
    "backsolve_transposed": ("s -= L[(size_t)b * rank + a] * W[(size_t)b * w + c];",
                             "s -= L[(size_t)a * rank + b] * W[(size_t)b * w + c];"),
    "values_beta": ("const double h = exp(beta * dot(ks, K + (size_t)i * d, d));",
                    "const double h = exp(0.5 * beta * dot(ks, K + (size_t)i * d, d));"),
    "no_rownorm": ("out[(size_t)q * dv + c] = A[c] / A[dv];", "out[(size_t)q * dv + c] = A[c];"),
    "no_stop_rule": ("int stop = dg[s] <= thresh;", "int stop = 0;"),
    "column_no_scale": ("Fi[j] = g / root;", "Fi[j] = g / dg[s];"),
}


def _build(name, tmpdir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmpdir, f"lib_{name}.so")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-I",
                    os.path.join(ROOT, "oracle"), path, "-o", so, "-lm"], check=True)
    return so


def _run_pins(so):
    env = dict(os.environ, WC_ORACLE_LIB=so)
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", *PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return p.returncode


def test_every_planted_mistake_fails_a_pin(tmp_path):
    names = sorted(MUTANTS)
    sos = [_build(n, str(tmp_path)) for n in names]
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        codes = list(ex.map(_run_pins, sos))
    survived = [n for n, c in zip(names, codes) if c == 0]
    assert not survived, f"mutants not caught by any pin: {survived}"
