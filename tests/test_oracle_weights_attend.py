"""Pins for the oracle's Nystrom weights, coreset attention and exact attention.

Independent checks:
  * W equals numpy's pseudo-inverse form pinv(H[S,S]) H[S,:] [V|1] (WildCat,
    gist.science technical summary, "Methodik" item 2), and the identity
    W = L^-T (F^T [V|1]) that follows from F = H[:,S] L^-T;
  * exact attention equals torch's scaled_dot_product_attention in fp64;
  * with r = n (or r at least the numerical rank) coreset attention equals
    exact attention (the optimal weights reconstruct the kernel exactly);
  * all keys equal: one pivot, and the output is the mean of V;
  * the error against exact attention falls as r grows (Abstract: error
    decays with the coreset size), median over seeds.
"""

import numpy as np
import pytest
import torch

import oracle


def kernel(A, B, beta):
    return np.exp(beta * np.asarray(A) @ np.asarray(B).T)


def problem(n, d, dv, nq, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((nq, d)) * scale, rng.standard_normal((n, d)) * scale,
            rng.standard_normal((n, dv)))


@pytest.mark.parametrize("n,d,dv,r,seed", [(30, 4, 3, 8, 0), (120, 8, 5, 20, 1), (64, 6, 4, 64, 2)])
def test_weights_match_pinv_and_factor_identity(n, d, dv, r, seed):
    Q, K, V = problem(n, d, dv, 5, seed)
    beta = 1.0 / np.sqrt(d)
    res = oracle.rpcholesky(K, r, beta, seed=seed, unit=0, eps_stop=1e-12)
    k = res["rank"]
    piv = res["piv"][:k]
    W = oracle.nystrom_weights(K, V, piv, k, beta)
    V1 = np.concatenate([V, np.ones((n, 1))], axis=1)
    Hss = kernel(K[piv], K[piv], beta)
    Hsk = kernel(K[piv], K, beta)
    C1 = oracle.coreset_values(K, V, piv, k, beta)
    assert np.allclose(C1, Hsk @ V1, rtol=1e-12, atol=0)
    Wp = np.linalg.pinv(Hss, rcond=1e-15, hermitian=True) @ Hsk @ V1
    cond = np.linalg.cond(Hss)
    assert np.max(np.abs(W - Wp)) <= 1e-13 * cond * np.max(np.abs(Wp))
    # identity form from the factor: W = L^-T (F^T [V|1])
    from scipy.linalg import solve_triangular

    F = res["F"][:, :k]
    L = F[piv, :]
    W2 = solve_triangular(L.T, F.T @ V1, lower=False)
    assert np.max(np.abs(W - W2)) <= 1e-12 * cond * np.max(np.abs(W))


@pytest.mark.parametrize("nq,nk,d,dv", [(7, 13, 4, 3), (33, 50, 16, 8), (5, 200, 64, 64)])
def test_exact_attention_matches_torch_sdpa(nq, nk, d, dv):
    Q, K, V = problem(nk, d, dv, nq, nq + nk, scale=1.0)
    beta = 0.37
    got = oracle.exact_attention(Q, K, V, beta)
    t = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))[None, None]
    want = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), scale=beta)[0, 0].numpy()
    assert np.max(np.abs(got - want)) <= 1e-12


@pytest.mark.parametrize("n,d,seed", [(12, 2, 0), (16, 4, 1), (10, 4, 2)])
def test_full_coreset_is_exact_attention(n, d, seed):
    Q, K, V = problem(n, d, 3, 9, seed, scale=0.8)
    beta = 1.0 / np.sqrt(d)
    res = oracle.rpcholesky(K, n, beta, seed=seed, unit=0, eps_stop=1e-13)
    assert res["rank"] == n
    piv = res["piv"]
    W = oracle.nystrom_weights(K, V, piv, n, beta)
    out = oracle.coreset_attend(Q, K[piv], W, beta)
    ex = oracle.exact_attention(Q, K, V, beta)
    assert np.max(np.abs(out - ex)) <= 1e-9


def test_rank_deficient_keys_give_exact_attention():
    rng = np.random.default_rng(3)
    m, d, reps = 4, 5, 6
    base = rng.standard_normal((m, d)) * 0.7
    K = base[rng.permutation(np.repeat(np.arange(m), reps))]
    V = rng.standard_normal((len(K), 3))
    Q = rng.standard_normal((6, d))
    beta = 1.0 / np.sqrt(d)
    res = oracle.rpcholesky(K, 12, beta, seed=1, unit=0)
    k = res["rank"]
    assert k == m
    W = oracle.nystrom_weights(K, V, res["piv"], k, beta)
    out = oracle.coreset_attend(Q, K[res["piv"][:k]], W, beta)
    assert np.max(np.abs(out - oracle.exact_attention(Q, K, V, beta))) <= 1e-8


def test_all_keys_equal_gives_mean_of_values():
    K = np.tile(np.array([[0.2, -0.4, 0.1]]), (20, 1))
    V = np.random.default_rng(0).standard_normal((20, 4))
    Q = np.random.default_rng(1).standard_normal((3, 3))
    res = oracle.rpcholesky(K, 5, 0.6, seed=0, unit=0)
    assert res["rank"] == 1
    W = oracle.nystrom_weights(K, V, res["piv"], 1, 0.6)
    out = oracle.coreset_attend(Q, K[res["piv"][:1]], W, 0.6)
    assert np.allclose(out, np.tile(V.mean(0), (3, 1)), rtol=0, atol=1e-12)


def test_error_falls_as_coreset_grows():
    n, d, dv = 64, 8, 4
    beta = 1.0 / np.sqrt(d)
    rs = [1, 2, 4, 8, 16, 32, 64]
    errs = np.zeros((32, len(rs)))
    for s in range(32):
        Q, K, V = problem(n, d, dv, 16, 100 + s, scale=0.6)
        ex = oracle.exact_attention(Q, K, V, beta)
        for a, r in enumerate(rs):
            res = oracle.rpcholesky(K, r, beta, seed=s, unit=0, eps_stop=1e-13)
            k = res["rank"]
            W = oracle.nystrom_weights(K, V, res["piv"], k, beta)
            out = oracle.coreset_attend(Q, K[res["piv"][:k]], W, beta)
            errs[s, a] = np.max(np.abs(out - ex))
    med = np.median(errs, axis=0)
    assert np.all(np.diff(med) <= 1e-12), med
    assert med[-1] <= 1e-8


def test_batched_forward_gqa_mapping():
    # forward() must send query head g to kv head g // (Hq/Hkv)
    rng = np.random.default_rng(5)
    B, Hq, Hkv, n, nq, d, dv, r = 2, 4, 2, 20, 6, 4, 3, 20
    Q = torch.from_numpy(rng.standard_normal((B, Hq, nq, d)) * 0.5)
    K = torch.from_numpy(rng.standard_normal((B, Hkv, n, d)) * 0.5)
    V = torch.from_numpy(rng.standard_normal((B, Hkv, n, dv)))
    res = oracle.forward(Q, K, V, r, seed=3, eps_stop=1e-13)
    beta = 1.0 / np.sqrt(d)
    for b in range(B):
        for g in range(Hq):
            h = g // (Hq // Hkv)
            ex = oracle.exact_attention(Q[b, g], K[b, h], V[b, h], beta)
            assert np.max(np.abs(res["out"][b, g] - ex)) <= 1e-8
