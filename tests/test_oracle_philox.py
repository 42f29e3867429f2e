"""Pins for the oracle's Philox4x32-10 and the pivot uniform.

The oracle's Philox is written from Salmon et al. (SC'11).  It is pinned here
against an independent library implementation: cuRAND's host-side
PHILOX4_32_10 generator, which runs on the CPU.  That generator emits the
output block of counter (x, y, z, 0) at element 4 * (65536 * P + z) where the
64-bit position P = y * 2^32 + x (65536 interleaved subsequences numbered by
the third counter word), so a generator offset selects any counter we need.
"""

import ctypes
import os

import numpy as np
import pytest

import oracle

CURAND = "/usr/local/cuda/lib64/libcurand.so"
PHILOX = 161  # CURAND_RNG_PSEUDO_PHILOX4_32_10


def _curand():
    if not os.path.exists(CURAND):
        pytest.skip("libcurand not available")
    lib = ctypes.CDLL(CURAND)
    lib.curandCreateGeneratorHost.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
    lib.curandSetPseudoRandomGeneratorSeed.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong]
    lib.curandSetGeneratorOffset.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong]
    lib.curandGenerate.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint), ctypes.c_size_t]
    lib.curandDestroyGenerator.argtypes = [ctypes.c_void_p]
    return lib


def _curand_block(lib, seed, x, y, z):
    g = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(g), PHILOX) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(g, seed) == 0
        pos = (y << 32) | x
        assert lib.curandSetGeneratorOffset(g, 4 * (65536 * pos + z)) == 0
        buf = (ctypes.c_uint * 4)()
        assert lib.curandGenerate(g, buf, 4) == 0
        return np.array(list(buf), dtype=np.uint32)
    finally:
        lib.curandDestroyGenerator(g)


@pytest.mark.parametrize(
    "seed,x,y,z",
    [
        (0, 0, 0, 0),
        (0, 1, 0, 0),
        (0, 5, 7, 0),
        (0x123456789ABCDEF, 3, 0, 11),
        (0xFEDCBA9876543210, 2047, 767, 0),
        (0xFFFFFFFFFFFFFFFF, 0xFFFFFFFF, 0x3FFF, 65535),  # offset must stay below 2^64
        (42, 131071, 3, 1),
    ],
)
def test_philox_matches_curand_host(seed, x, y, z):
    lib = _curand()
    want = _curand_block(lib, seed, x, y, z)
    got = oracle.philox4x32_10([x, y, z, 0], [seed & 0xFFFFFFFF, seed >> 32])
    assert np.array_equal(got, want), (got, want)


def test_pivot_uniform_is_first_word_over_2_32():
    for seed, j, unit in [(0, 0, 0), (0, 17, 3), (2**63 + 5, 2047, 767)]:
        w = oracle.philox4x32_10([j, unit, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        u = oracle.pivot_uniform(seed, j, unit)
        assert u == float(w[0]) / 2.0**32
        assert 0.0 <= u < 1.0


def test_pivot_uniforms_are_uniform():
    # Kolmogorov-Smirnov against U[0,1) over 20000 (step, unit) counters.
    from scipy import stats

    us = np.array([oracle.pivot_uniform(7, j, u) for u in range(10) for j in range(2000)])
    assert stats.kstest(us, "uniform").pvalue > 1e-3
