"""Pins of the oracle's binned selection and key centring (the method's
divide-and-conquer selection, WildCat gist.science summary "Methodik" item 1
"Effizienz", and its centring, item 3), against closed forms and invariants
that a wrong bin bookkeeping or a missing centring would break."""

from __future__ import annotations

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _inputs(seed, B=1, H=2, n=16, nq=5, d=4, dv=3, scale=0.6):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, nq, d)) * scale
    K = rng.standard_normal((B, H, n, d)) * scale
    V = rng.standard_normal((B, H, n, dv))
    return Q, K, V


def _exact(Q, K, V, beta):
    B, H = Q.shape[:2]
    out = np.zeros(Q.shape[:3] + (V.shape[-1],))
    for b in range(B):
        for h in range(H):
            out[b, h] = oracle.exact_attention(Q[b, h], K[b, h], V[b, h], beta)
    return out


@pytest.mark.parametrize("bins", [1, 2, 4])
def test_bins_with_every_key_selected_is_exact_attention(bins):
    # r = n: every bin's Nystrom step is exact on its own keys, so the union of
    # the bins' weighted coresets reproduces softmax attention over all keys.
    Q, K, V = _inputs(1)
    n = K.shape[2]
    o = oracle.forward(Q, K, V, n, seed=3, eps_stop=1e-13, bins=bins)
    ref = _exact(Q, K, V, o["beta"])
    assert np.max(np.abs(o["out"] - ref)) <= 1e-8 * np.max(np.abs(ref))
    if bins > 1:
        assert o["rank"].shape == (1, 2, bins) and np.all(o["rank"] == n // bins)


def test_bins_rank_deficient_bins_are_exact():
    # Each bin holds 3 distinct keys, repeated: the bin's selection stops at
    # rank 3 and the union of the bins' coresets is still exact attention.
    rng = np.random.default_rng(5)
    bins, nb, d, dv = 2, 12, 4, 3
    K = np.zeros((1, 1, bins * nb, d))
    for b in range(bins):
        distinct = rng.standard_normal((3, d)) * 0.7
        K[0, 0, b * nb:(b + 1) * nb] = distinct[rng.integers(0, 3, nb) if b else np.arange(nb) % 3]
    Q = rng.standard_normal((1, 1, 6, d)) * 0.7
    V = rng.standard_normal((1, 1, bins * nb, dv))
    o = oracle.forward(Q, K, V, 8, seed=2, bins=bins)
    assert np.all(o["rank"] == 3)
    piv = o["piv"][0, 0]
    for b in range(bins):
        got = piv[b * 4:(b + 1) * 4]
        assert np.all((got[:3] >= b * nb) & (got[:3] < (b + 1) * nb)) and got[3] == -1
    ref = _exact(Q, K, V, o["beta"])
    assert np.max(np.abs(o["out"] - ref)) <= 1e-8 * np.max(np.abs(ref))


def test_bins_first_pivot_follows_the_bin_diagonal():
    # The first pivot of bin b is drawn with probability exp(beta |k_i|^2) /
    # sum over the bin's keys (its own Philox stream, unit index u * bins + b):
    # a chi-square test over many seeds for bin 1 of unit 0.
    rng = np.random.default_rng(11)
    bins, nb, d = 2, 6, 3
    K = rng.standard_normal((1, 1, bins * nb, d)) * 0.8
    Q = rng.standard_normal((1, 1, 1, d))
    V = rng.standard_normal((1, 1, bins * nb, 2))
    beta = oracle.default_beta(d)
    dg = np.exp(beta * np.sum(K[0, 0, nb:] ** 2, axis=1))
    p = dg / dg.sum()
    counts = np.zeros(nb)
    trials = 3000
    for seed in range(trials):
        res = oracle.rpcholesky(K[0, 0, nb:], 1, beta, seed=seed, unit=0 * bins + 1)
        counts[res["piv"][0]] += 1
    chi2 = np.sum((counts - trials * p) ** 2 / (trials * p))
    assert chi2 < 25.0  # 5 degrees of freedom: p-value ~ 1e-4
    # and the binned forward draws bin 1's first pivot from that same stream
    o = oracle.forward(Q, K, V, 2, seed=7, bins=bins)
    one = oracle.rpcholesky(K[0, 0, nb:], 1, beta, seed=7, unit=1)
    assert o["piv"][0, 0, 1] == one["piv"][0] + nb


def test_bins_factor_is_block_diagonal_and_interpolates_each_bin():
    Q, K, V = _inputs(4, n=24)
    bins, r = 3, 6
    o = oracle.forward(Q, K, V, r, seed=1, bins=bins)
    beta = o["beta"]
    nb, rb = 8, 2
    for h in range(2):
        F = o["F"][0, h]
        for b in range(bins):
            blk = F[b * nb:(b + 1) * nb, b * rb:(b + 1) * rb]
            mask = np.ones_like(F, dtype=bool)
            mask[b * nb:(b + 1) * nb, b * rb:(b + 1) * rb] = False
            assert np.all(F[b * nb:(b + 1) * nb][mask[b * nb:(b + 1) * nb]] == 0.0)
            S = o["piv"][0, h, b * rb:(b + 1) * rb] - b * nb
            Kb = K[0, h, b * nb:(b + 1) * nb]
            H = np.exp(beta * Kb @ Kb.T)
            # F F^T reproduces the bin's kernel matrix on its pivot rows
            assert np.allclose((blk @ blk.T)[S], H[S], rtol=1e-10, atol=0)


def test_centring_is_invariant_to_a_common_key_offset():
    # Centred selection and weights see K - mean(K): adding one vector c to
    # every key changes nothing (pivots, W, output), while without centring
    # the same offset changes the kernel matrix and the run.
    Q, K, V = _inputs(8, n=20, d=4)
    c = np.array([1.5, -2.0, 0.7, 3.0])
    K2 = K + c
    a = oracle.forward(Q, K, V, 6, seed=4, center=True)
    b = oracle.forward(Q, K2, V, 6, seed=4, center=True)
    assert np.array_equal(a["piv"], b["piv"]) and np.array_equal(a["rank"], b["rank"])
    assert np.allclose(a["W"], b["W"], rtol=1e-9, atol=1e-12)
    assert np.allclose(a["out"], b["out"], rtol=1e-9, atol=1e-12)
    u = oracle.forward(Q, K, V, 6, seed=4)
    u2 = oracle.forward(Q, K2, V, 6, seed=4)
    assert not np.allclose(u["W"], u2["W"], rtol=1e-3)


def test_centring_with_every_key_selected_is_exact_attention():
    Q, K, V = _inputs(9, n=12, d=3)
    K = K + np.array([0.8, -0.5, 1.2])
    o = oracle.forward(Q, K, V, 12, seed=0, eps_stop=1e-13, center=True)
    ref = _exact(Q, K, V, o["beta"])
    assert np.max(np.abs(o["out"] - ref)) <= 1e-8 * np.max(np.abs(ref))


def test_centring_factor_interpolates_the_centred_kernel():
    Q, K, V = _inputs(10, n=18, d=4)
    K = K + 0.9
    o = oracle.forward(Q, K, V, 5, seed=6, center=True)
    beta = o["beta"]
    for h in range(2):
        Kc = K[0, h] - K[0, h].mean(axis=0)
        H = np.exp(beta * Kc @ Kc.T)
        F = o["F"][0, h]
        S = o["piv"][0, h][: o["rank"][0, h]]
        assert np.allclose((F @ F.T)[S], H[S], rtol=1e-10, atol=0)
        Hraw = np.exp(beta * K[0, h] @ K[0, h].T)
        assert not np.allclose((F @ F.T)[S], Hraw[S], rtol=1e-3)
