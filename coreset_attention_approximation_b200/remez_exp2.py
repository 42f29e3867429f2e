"""Minimax polynomial for 2^f on [-1/2, 1/2], fitted by the Remez exchange
algorithm (E. Ya. Remez, 1934; see e.g. J.-M. Muller, "Elementary Functions:
Algorithms and Implementation", ch. 3), minimising the RELATIVE error.

The tensor-core exp-GEMM computes part of its exponentials on the FMA / ALU
pipes instead of the exponential unit (csrc/wc_exp2.cuh): an additive range
reduction x = n + f with n = rint(x) (Cody and Waite's scheme, W. J. Cody and
W. Waite, "Software Manual for the Elementary Functions", 1980; for base 2 the
reduction is exact, no split constant is needed), 2^f by the polynomial below,
and 2^n added to the exponent field.  This script derives the polynomial's
coefficients; the header holds them as fp32 hexadecimal literals, and
tests/test_exp2_poly.py checks that the two agree and that the fp32
evaluation meets the stated error bound.

    python -m coreset_attention_approximation_b200.remez_exp2 [degree]
"""

from __future__ import annotations

import sys

import numpy as np


def remez(degree: int, a: float = -0.5, b: float = 0.5, iters: int = 40, grid: int = 200001):
    """Coefficients c[0..degree] (lowest power first) of the polynomial p that
    minimises max |p(f) - 2^f| / 2^f on [a, b], and that maximum.

    Each iteration solves p(x_i) - 2^x_i = (-1)^i E 2^x_i on degree + 2
    reference points (the equioscillation conditions), then moves the
    reference to the extrema of the error in each interval where its sign is
    constant, until the extrema level out at |E|."""
    n = degree + 2
    k = np.arange(n)
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * k / (n - 1))   # Chebyshev extrema, ascending
    g = np.linspace(a, b, grid)
    fg = np.exp2(g)
    c = None
    for _ in range(iters):
        A = np.empty((n, n))
        A[:, : degree + 1] = x[:, None] ** np.arange(degree + 1)[None, :]
        A[:, degree + 1] = (-1.0) ** k * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[: degree + 1]
        err = (np.polynomial.polynomial.polyval(g, c) - fg) / fg
        sign_change = np.where(np.diff(np.sign(err)) != 0)[0]
        segments = np.split(np.arange(grid), sign_change + 1)
        pts = [s[np.argmax(np.abs(err[s]))] for s in segments]
        if len(pts) > n:   # keep the n largest, in order
            pts = sorted(sorted(pts, key=lambda i: -abs(err[i]))[:n])
        if len(pts) == n:
            x = g[pts]
    err = (np.polynomial.polynomial.polyval(g, c) - fg) / fg
    return c, float(np.abs(err).max())


def _hex32(v: float) -> str:
    """C hexadecimal literal of v rounded to fp32 (e.g. 0x1.62e43p-1f)."""
    f = float(np.float32(v))
    mant, exp = f.hex().split("p")
    mant = mant.rstrip("0")
    if mant.endswith("."):
        mant = mant[:-1]
    return f"{mant}p{int(exp)}f"


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    degree = int(argv[0]) if argv else 3
    c, e = remez(degree)
    print(f"// degree {degree}, max relative error {e:.3e} (2^{np.log2(e):.2f}) on [-1/2, 1/2]")
    for i, v in enumerate(c):
        print(f"constexpr float kExp2C{i} = {_hex32(v)};")
    return 0


if __name__ == "__main__":
    sys.exit(main())
