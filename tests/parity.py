"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare them."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from coreset_attention_approximation_b200 import wildcat

TOL_OUT = {torch.float32: 1e-5, torch.bfloat16: 2e-3}


def rel_err(got, want) -> float:
    """max |got - want| / max |want| (the relative error the tests bound)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.max(np.abs(want))
    return float(np.max(np.abs(got - want)) / den) if den > 0 else float(np.max(np.abs(got)))


def factor_shift(K, beta, center=False) -> float:
    """M = max_i beta |k_i|^2 of one unit's (or bin's) keys: the library's F is
    the factor of exp(beta K K^T - M), the oracle's F times exp(-M / 2)."""
    Kd = np.asarray(K, dtype=np.float64)
    if center:
        Kd = Kd - Kd.mean(axis=0, keepdims=True)
    return float(beta * np.max(np.sum(Kd * Kd, axis=1)))


def run_gpu(Q, K, V, r, seed=0, **kw):
    dev = torch.device("cuda")
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    res = wildcat.forward(Qd, Kd, Vd, r, seed=seed, **kw)
    torch.cuda.synchronize()
    status = wildcat.check_device_status(res["ws"])
    assert status == 0, wildcat.STATUS.get(status, status)
    return {k: v.cpu() for k, v in res.items() if k != "ws"}


def compare(Q, K, V, r, seed=0, eps_stop=None, check_F=True, tol_w=None, units=None, **kw):
    """GPU forward vs oracle forward (pivots replayed within the 1e-6 window).
    units: optional list of (batch * Hkv + kv-head) indices the oracle checks
    (the GPU still runs every unit); the outputs checked are those of the query
    heads of those units.  Returns a dict of the measured errors; asserts the
    tolerances."""
    gkw = dict(kw)
    okw = {}
    if eps_stop is not None:
        gkw["eps_stop"] = eps_stop
        okw["eps_stop"] = float(np.float32(eps_stop))
    g = run_gpu(Q, K, V, r, seed=seed, **gkw)
    piv_g, rank_g = g["piv"].numpy(), g["rank"].numpy()
    o = oracle.forward(Q, K, V, r, seed=seed, replay=(piv_g, rank_g), units=units, **okw)
    B, Hkv = rank_g.shape
    n = K.shape[2]
    checked = set(range(B * Hkv)) if units is None else set(units)
    report = dict(replays=0, max_margin=0.0, err_out=0.0, err_W=0.0, err_F=0.0)
    for b in range(B):
        for h in range(Hkv):
            if b * Hkv + h not in checked:
                continue
            info = o["info"][b * Hkv + h]
            assert info["failed_step"] == -1, (b, h, info)
            report["replays"] += info["n_replays"]
            report["max_margin"] = max(report["max_margin"], info["max_margin"])
            k = int(rank_g[b, h])
            assert k == int(o["rank"][b, h])
            assert np.array_equal(piv_g[b, h], o["piv"][b, h])
            if check_F:
                Fg = g["F"][b, h].numpy()[:, :n].T          # n x r
                M = factor_shift(K[b, h].double().numpy(), o["beta"])
                report["err_F"] = max(report["err_F"], rel_err(Fg, o["F"][b, h] * np.exp(-M / 2)))
                assert np.all(g["F"][b, h].numpy()[:, n:] == 0.0)
            if k > 0:
                report["err_W"] = max(report["err_W"], rel_err(g["W"][b, h].numpy()[:k], o["W"][b, h, :k]))
            assert np.all(g["W"][b, h].numpy()[k:] == 0.0)
    tol = TOL_OUT[K.dtype]
    group = Q.shape[1] // Hkv
    for b in range(B):
        for hq in range(Q.shape[1]):
            if b * Hkv + hq // group not in checked:
                continue
            report["err_out"] = max(report["err_out"], rel_err(g["out"][b, hq].numpy(), o["out"][b, hq]))
    assert report["err_out"] <= tol, report
    if check_F:
        assert report["err_F"] <= 1e-5, report
    if tol_w is not None:
        assert report["err_W"] <= tol_w, report
    return report


def compare_next(Q, K, V, r, seed=0, bins=1, center=False, check_F=True, tol_w=None, **kw):
    """compare() for the binned selection and key centring: per-bin pivots,
    ranks and factors against the oracle's (replayed within the 1e-6 window),
    W and the output within the dtype's tolerance."""
    g = run_gpu(Q, K, V, r, seed=seed, bins=bins, center=center, **kw)
    piv_g, rank_g = g["piv"].numpy(), g["rank"].numpy()
    nb = max(bins, 1)
    rank3 = rank_g.reshape(rank_g.shape[0], rank_g.shape[1], nb)
    o = oracle.forward(Q, K, V, r, seed=seed, replay=(piv_g, rank3), bins=nb, center=center)
    B, Hkv = rank3.shape[:2]
    n = K.shape[2]
    nbk, rb = n // nb, r // nb
    orank = np.asarray(o["rank"]).reshape(B, Hkv, nb)
    report = dict(replays=0, err_out=0.0, err_W=0.0, err_F=0.0)
    for b in range(B):
        for h in range(Hkv):
            for bb in range(nb):
                info = o["info"][(b * Hkv + h) * nb + bb]
                assert info["failed_step"] == -1, (b, h, bb, info)
                report["replays"] += info["n_replays"]
                k = int(rank3[b, h, bb])
                assert k == int(orank[b, h, bb]), (b, h, bb)
                if check_F:
                    Fg = g["F"][b, h].numpy().reshape(nb, rb, -1)[bb][:, :nbk].T if nb > 1 else \
                        g["F"][b, h].numpy()[:, :n].T
                    Kc = K[b, h].double().numpy()
                    if center:
                        Kc = Kc - Kc.mean(axis=0, keepdims=True)
                    M = factor_shift(Kc[bb * nbk:(bb + 1) * nbk], o["beta"])
                    Fo = o["F"][b, h, bb * nbk:(bb + 1) * nbk, bb * rb:(bb + 1) * rb] * np.exp(-M / 2)
                    report["err_F"] = max(report["err_F"], rel_err(Fg, Fo))
                rows = slice(bb * rb, bb * rb + k)
                if k > 0:
                    report["err_W"] = max(report["err_W"], rel_err(g["W"][b, h].numpy()[rows], o["W"][b, h, rows]))
                assert np.all(g["W"][b, h].numpy()[bb * rb + k:(bb + 1) * rb] == 0.0)
            assert np.array_equal(piv_g[b, h], o["piv"][b, h])
    tol = TOL_OUT[K.dtype]
    for b in range(B):
        for hq in range(Q.shape[1]):
            report["err_out"] = max(report["err_out"], rel_err(g["out"][b, hq].numpy(), o["out"][b, hq]))
    assert report["err_out"] <= tol, report
    if check_F:
        assert report["err_F"] <= 1e-5, report
    if tol_w is not None:
        assert report["err_W"] <= tol_w, report
    return report
