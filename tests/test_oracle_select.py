"""Pins for the oracle's randomly pivoted Cholesky.

What fixes the result independently of the oracle's own code:
  * the sampling law: a pivot is drawn with probability proportional to the
    current residual diagonal (WildCat, gist.science technical summary,
    "Methodik" item 1) — checked by a chi-square test over many seeds, at the
    first step (p_i ~ H_ii) and the second (p_k ~ H_kk - H_ks^2 / H_ss);
  * Cholesky algebra: the residual trace equals trace(H) - |F|_F^2, F F^T
    reproduces H on the pivot rows, F[S,:] is lower triangular and equals the
    textbook Cholesky factor of H[S,S] (numpy), F = H[:,S] F[S,:]^-T;
  * the residual of a positive semidefinite matrix has a non-negative diagonal;
  * rank deficiency: keys with m distinct rows make H rank m, so the run stops
    at rank m with one pivot per distinct row.
"""

import numpy as np
import pytest
from scipy import stats

import oracle


def kernel(K, beta):
    K = np.asarray(K, dtype=np.float64)
    return np.exp(beta * K @ K.T)


def rand_keys(n, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((n, d)) * scale


@pytest.mark.parametrize("n,d,r,seed", [(40, 4, 12, 0), (200, 8, 30, 1), (64, 16, 64, 2), (1000, 64, 40, 3)])
def test_cholesky_invariants(n, d, r, seed):
    K = rand_keys(n, d, seed, scale=0.5)
    beta = 1.0 / np.sqrt(d)
    H = kernel(K, beta)
    res = oracle.rpcholesky(K, r, beta, seed=seed, unit=seed, eps_stop=1e-13)
    k = res["rank"]
    piv = res["piv"][:k]
    F = res["F"][:, :k]
    scale = np.trace(H)
    assert len(set(piv.tolist())) == k                      # distinct pivots
    assert np.all(res["piv"][k:] == -1)
    assert np.all(res["F"][:, k:] == 0.0)
    # residual trace: sum(d) before step j = trace(H) - |F[:, :j]|_F^2
    for j in range(k + 1):
        want = np.trace(H) - np.sum(F[:, :j] ** 2)
        assert abs(res["dsum"][j] - want) <= 1e-10 * scale
    # interpolation on the pivot rows
    assert np.max(np.abs((F @ F.T)[piv, :] - H[piv, :])) <= 1e-10 * H.max()
    # lower-triangular pivot rows with positive diagonal
    L = F[piv, :]
    assert np.all(np.triu(L, 1) == 0.0)
    assert np.all(np.diag(L) > 0.0)
    # textbook Cholesky of H[S,S] (numpy)
    Lnp = np.linalg.cholesky(H[np.ix_(piv, piv)])
    assert np.max(np.abs(L - Lnp)) <= 1e-10 * np.sqrt(H.max())
    # F = H[:, S] L^-T
    from scipy.linalg import solve_triangular

    F2 = solve_triangular(L, H[:, piv].T, lower=True).T
    assert np.max(np.abs(F - F2)) <= 1e-9 * np.sqrt(H.max())
    # the residual diagonal never went below zero beyond rounding
    assert res["dneg"] >= -1e-12


def _first_two_pivots(K, beta, seeds):
    s0 = np.empty(len(seeds), dtype=np.int64)
    s1 = np.empty(len(seeds), dtype=np.int64)
    for a, sd in enumerate(seeds):
        res = oracle.rpcholesky(K, 2, beta, seed=int(sd), unit=0, eps_stop=0.0)
        s0[a], s1[a] = res["piv"][0], res["piv"][1]
    return s0, s1


def test_sampling_law_first_and_second_pivot():
    n, d = 8, 3
    K = rand_keys(n, d, 11, scale=0.8)
    beta = 1.0 / np.sqrt(d)
    H = kernel(K, beta)
    seeds = [(a * 0x9E3779B97F4A7C15) % 2**64 for a in range(40000)]
    s0, s1 = _first_two_pivots(K, beta, seeds)
    # step 0: p_i = H_ii / trace(H)
    p0 = np.diag(H) / np.trace(H)
    obs = np.bincount(s0, minlength=n)
    assert stats.chisquare(obs, p0 * len(seeds)).pvalue > 1e-4
    # step 1 given s0 = a: p_k ~ H_kk - H_ka^2 / H_aa (zero at k = a)
    a = int(np.argmax(obs))
    sel = s1[s0 == a]
    res1 = np.diag(H) - H[:, a] ** 2 / H[a, a]
    res1[a] = 0.0
    p1 = res1 / res1.sum()
    obs1 = np.bincount(sel, minlength=n)
    keep = p1 > 0
    assert obs1[~keep].sum() == 0
    assert stats.chisquare(obs1[keep], p1[keep] * len(sel)).pvalue > 1e-4


def test_inverse_cdf_boundaries_equal_diagonal():
    # All H_ii equal (unit-norm keys): step 0 picks floor(u * n) exactly.
    n, d = 37, 5
    K = rand_keys(n, d, 5)
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    for seed in range(30):
        u = oracle.pivot_uniform(seed, 0, 4)
        res = oracle.rpcholesky(K, 1, 0.7, seed=seed, unit=4)
        want = int(np.floor(u * n))
        # guard against a draw that sits on a boundary within rounding
        if abs(u * n - round(u * n)) > 1e-9:
            assert res["piv"][0] == want


def test_inverse_cdf_rule_on_exact_ties():
    # smallest i with C_i > t (strict): a zero-width interval is never drawn,
    # and t on a boundary goes to the next interval with positive width.
    dg = [1.0, 0.0, 2.0, 0.0, 0.0, 1.0]
    assert oracle.inverse_cdf(dg, 0.0) == 0
    assert oracle.inverse_cdf(dg, 0.5) == 0
    assert oracle.inverse_cdf(dg, 1.0) == 2
    assert oracle.inverse_cdf(dg, 2.999) == 2
    assert oracle.inverse_cdf(dg, 3.0) == 5
    assert oracle.inverse_cdf([0.0, 0.0, 4.0], 0.0) == 2
    # t at or above the total (only reachable through rounding): last positive
    assert oracle.inverse_cdf(dg, 4.0) == 5
    assert oracle.inverse_cdf([0.0, 3.0, 0.0], 5.0) == 1
    assert oracle.inverse_cdf([0.0, 0.0], 0.0) == -1


def test_rank_deficient_keys_stop_at_numerical_rank():
    rng = np.random.default_rng(4)
    m, d, reps = 5, 6, 9
    base = rng.standard_normal((m, d)) * 0.6
    idx = rng.permutation(np.repeat(np.arange(m), reps))
    K = base[idx]
    res = oracle.rpcholesky(K, 20, 1.0 / np.sqrt(d), seed=3, unit=0)
    assert res["rank"] == m
    assert sorted(idx[res["piv"][:m]].tolist()) == list(range(m))


def test_all_keys_equal_rank_one():
    K = np.tile(np.array([[0.3, -0.2, 0.5, 0.1]]), (16, 1))
    res = oracle.rpcholesky(K, 4, 0.5, seed=1, unit=0)
    assert res["rank"] == 1


def test_r_equals_n_exhausts_trace():
    K = rand_keys(24, 4, 8, scale=0.7)
    res = oracle.rpcholesky(K, 24, 0.5, seed=2, unit=1, eps_stop=1e-13)
    H = kernel(K, 0.5)
    assert res["rank"] == 24
    assert res["dsum"][-1] <= 1e-10 * np.trace(H)


def test_replay_accepts_within_window_and_refuses_outside():
    n, d = 50, 4
    K = rand_keys(n, d, 9, scale=0.3)
    beta = 0.5
    own = oracle.rpcholesky(K, 10, beta, seed=5, unit=2)
    same = oracle.rpcholesky(K, 10, beta, seed=5, unit=2, replay_piv=own["piv"], replay_rank=own["rank"])
    assert same["n_replays"] == 0 and same["failed_step"] == -1
    assert np.array_equal(same["piv"], own["piv"])
    # move the pivot of step 3 to a far index: refused with window 1e-6 ...
    alt = own["piv"].copy()
    far = int((alt[3] + n // 2) % n)
    while far in alt[:3]:
        far = (far + 1) % n
    alt[3] = far
    bad = oracle.rpcholesky(K, 10, beta, seed=5, unit=2, replay_piv=alt, replay_rank=own["rank"])
    assert bad["failed_step"] == 3 and bad["fail_margin"] > 1e-6
    # ... and accepted when the window covers the whole CDF
    # (the replayed run stops after step 3; the stop decision is replayed too)
    alt[4:] = -1
    ok = oracle.rpcholesky(K, 10, beta, seed=5, unit=2, replay_piv=alt, replay_rank=4, window=1.0)
    assert ok["failed_step"] == -1 and ok["n_replays"] == 2 and ok["rank"] == 4 and ok["piv"][3] == far
    # margin closed form at step 0 with equal diagonal: boundaries at k * T / n
    Ku = K / np.linalg.norm(K, axis=1, keepdims=True)
    u = oracle.pivot_uniform(5, 0, 2)
    s0 = int(np.floor(u * n))
    alt0 = np.full(10, -1, dtype=np.int32)
    alt0[0] = (s0 + 2) % n if s0 + 2 < n else s0 - 2
    res = oracle.rpcholesky(Ku, 10, beta, seed=5, unit=2, replay_piv=alt0, replay_rank=10)
    other = alt0[0]
    want = ((other) / n - u) if other > s0 else (u - (other + 1) / n)
    assert res["failed_step"] == 0
    assert abs(res["fail_margin"] - want) < 1e-12
