"""The exp-GEMM's exponential on the FMA / ALU pipes (csrc/wc_exp2.cuh).

Pinned from outside the kernel code: the header's coefficients are the Remez
fit that remez_exp2.py computes (rounded to fp32), the fit equioscillates as a
minimax polynomial must (Chebyshev's alternation theorem), and an fp32
emulation of the header's steps meets the stated relative error bound against
2^x in fp64.  The GPU tests run the device function itself through
wc_selftest_exp2 against 2^x (fp64), CUDA's exp2f (torch.exp2) and the CPU
emulation.
"""

from __future__ import annotations

import os
import re

import numpy as np
import pytest

from coreset_attention_approximation_b200 import remez_exp2

HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(HERE, "..", "coreset_attention_approximation_b200", "csrc", "wc_exp2.cuh")
BOUND = 2.0 ** -13.5     # relative error the header states for -125 <= x <= 127
ULP_BOUND = 1500         # the same bound in fp32 ulps of the result (2^-13.5 * 2^24 = 1448)


def header_constants():
    text = open(HEADER).read()
    vals = dict(re.findall(r"constexpr float (kExp2\w+) = ([-0-9a-fx.p+]+)f;", text))
    return {k: float.fromhex(v) if "0x" in v else float(v) for k, v in vals.items()}


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def _fma32(a, b, c):
    # a*b is exact in fp64 (24 + 24 bits); one fp64 add then one fp32 rounding
    return _f32(np.float64(a) * np.float64(b) + np.float64(c))


def emulate(x):
    """The header's steps in fp32 arithmetic (numpy rounds fp32 adds and
    products to nearest and keeps subnormals, as the device's .rn ops do)."""
    k = header_constants()
    x = np.maximum(_f32(x), np.float32(k["kExp2Lo"]))
    shift = np.float32(k["kExp2Shift"])
    t = _f32(x + shift)
    f = _f32(x - _f32(t - shift))
    p = _fma32(np.float32(k["kExp2C3"]), f, np.float32(k["kExp2C2"]))
    p = _fma32(p, f, np.float32(k["kExp2C1"]))
    p = _fma32(p, f, np.float32(k["kExp2C0"]))
    sbits = (t.view(np.uint32).astype(np.uint64) << np.uint64(23)) & np.uint64(0xFFFFFFFF)
    sc = sbits.astype(np.uint32).view(np.float32)
    return _f32(p * sc)


def sweep(n=2_000_001, lo=-125.0, hi=127.0, seed=0):
    rng = np.random.default_rng(seed)
    x = np.concatenate([np.linspace(lo, hi, n), rng.uniform(lo, hi, n // 2),
                        np.arange(-125, 128, dtype=np.float64),            # integers: f = 0
                        np.arange(-125, 127, dtype=np.float64) + 0.5,      # rounding ties of rint
                        rng.uniform(-1.0, 1.0, 100_000)])
    return _f32(x)


def test_header_coefficients_are_the_remez_fit():
    c, err = remez_exp2.remez(3)
    k = header_constants()
    for i in range(4):
        assert np.float32(c[i]) == np.float32(k[f"kExp2C{i}"]), i
    assert 7.0e-5 < err < 7.6e-5          # the fit's own maximum relative error (2^-13.71)
    assert k["kExp2Shift"] == 1.5 * 2 ** 23 + 127 and k["kExp2Lo"] == -127.0


def test_fit_equioscillates():
    """A minimax polynomial of degree 3 has an error curve with 5 extrema of
    equal size and alternating sign (Chebyshev alternation)."""
    c, err = remez_exp2.remez(3)
    g = np.linspace(-0.5, 0.5, 400001)
    e = (np.polynomial.polynomial.polyval(g, c) - np.exp2(g)) / np.exp2(g)
    inner = np.where((np.abs(e[1:-1]) >= np.abs(e[:-2])) & (np.abs(e[1:-1]) >= np.abs(e[2:])))[0] + 1
    ext = [0] + [i for i in inner if abs(e[i]) > 0.9 * err] + [len(g) - 1]
    vals = e[ext]
    assert len(ext) == 5, len(ext)
    assert np.all(np.sign(vals[1:]) == -np.sign(vals[:-1]))
    assert np.abs(vals).min() > 0.999 * np.abs(vals).max()


def test_higher_degree_fits_are_more_accurate():
    # the exchange itself, on its own terms: each added degree gains more than 4 bits
    errs = [remez_exp2.remez(d)[1] for d in (2, 3, 4, 5)]
    assert all(a > 20 * b for a, b in zip(errs, errs[1:])), errs


def test_fp32_steps_meet_the_stated_bound():
    x = sweep()
    y = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() <= BOUND, rel.max()
    assert rel.max() > 0.9 * 7.478e-5     # and the fit's error is really there (not an exact exp)


def test_underflow_is_small_and_ends_in_exact_zero():
    x = _f32(np.linspace(-127.0, -125.0, 20001))
    y = emulate(x).astype(np.float64)
    assert np.all(np.abs(y - np.exp2(x.astype(np.float64))) <= 2.0 ** -125)
    z = emulate(_f32([-127.0, -128.0, -1e4, -np.inf]))
    assert np.all(z == 0.0)


@pytest.mark.gpu
def test_gpu_polynomial_meets_the_bound_and_matches_the_emulation():
    import torch
    from coreset_attention_approximation_b200 import wildcat

    x = sweep()
    xd = torch.from_numpy(x).cuda()
    y = wildcat.selftest_exp2(xd, method=0).cpu().numpy()
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y.astype(np.float64) - ref) / ref
    assert rel.max() <= BOUND, rel.max()
    # against CUDA's exp2f, in ulps of exp2f's result
    e2 = torch.exp2(xd).cpu().numpy()
    ulp = np.spacing(np.abs(e2)).astype(np.float64)
    assert (np.abs(y.astype(np.float64) - e2) / ulp).max() <= ULP_BOUND
    # the device's fused multiply-adds round once; the emulation's at most twice
    em = emulate(x)
    diff = np.abs(y.view(np.int32).astype(np.int64) - em.view(np.int32).astype(np.int64))
    assert diff.max() <= 1 and (diff == 0).mean() > 0.9999
    # odd length (the last element computed alone) and the underflow to exact zero
    xs = torch.tensor([-3.25, 0.0, 1.0, -200.0, -float("inf"), 8.0, -126.0], device="cuda")
    ys = wildcat.selftest_exp2(xs, method=0).cpu().numpy().astype(np.float64)
    assert np.allclose(ys[[0, 1, 2, 5]], np.exp2([-3.25, 0.0, 1.0, 8.0]), rtol=BOUND, atol=0)
    assert ys[3] == 0.0 and ys[4] == 0.0 and abs(ys[6] - 2.0 ** -126) <= 2.0 ** -125


@pytest.mark.gpu
def test_gpu_exponential_unit_is_close_to_exp2():
    import torch
    from coreset_attention_approximation_b200 import wildcat

    x = sweep(n=200_001, lo=-126.0, hi=127.0)
    y = wildcat.selftest_exp2(torch.from_numpy(x).cuda(), method=1).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(y - ref) / ref).max() <= 2.0 ** -21
