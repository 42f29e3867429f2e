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


def run_gpu(Q, K, V, r, seed=0, **kw):
    dev = torch.device("cuda")
    Qd, Kd, Vd = Q.to(dev), K.to(dev), V.to(dev)
    res = wildcat.forward(Qd, Kd, Vd, r, seed=seed, **kw)
    torch.cuda.synchronize()
    status = wildcat.check_device_status(res["ws"])
    assert status == 0, wildcat.STATUS.get(status, status)
    return {k: v.cpu() for k, v in res.items() if k != "ws"}


def compare(Q, K, V, r, seed=0, eps_stop=None, check_F=True, tol_w=None, **kw):
    """GPU forward vs oracle forward (pivots replayed within the 1e-6 window).
    Returns a dict of the measured errors; asserts the tolerances."""
    gkw = dict(kw)
    okw = {}
    if eps_stop is not None:
        gkw["eps_stop"] = eps_stop
        okw["eps_stop"] = float(np.float32(eps_stop))
    g = run_gpu(Q, K, V, r, seed=seed, **gkw)
    piv_g, rank_g = g["piv"].numpy(), g["rank"].numpy()
    o = oracle.forward(Q, K, V, r, seed=seed, replay=(piv_g, rank_g), **okw)
    B, Hkv = rank_g.shape
    n = K.shape[2]
    report = dict(replays=0, max_margin=0.0, err_out=0.0, err_W=0.0, err_F=0.0)
    for b in range(B):
        for h in range(Hkv):
            info = o["info"][b * Hkv + h]
            assert info["failed_step"] == -1, (b, h, info)
            report["replays"] += info["n_replays"]
            report["max_margin"] = max(report["max_margin"], info["max_margin"])
            k = int(rank_g[b, h])
            assert k == int(o["rank"][b, h])
            assert np.array_equal(piv_g[b, h], o["piv"][b, h])
            if check_F:
                Fg = g["F"][b, h].numpy()[:, :n].T          # n x r
                report["err_F"] = max(report["err_F"], rel_err(Fg, o["F"][b, h]))
                assert np.all(g["F"][b, h].numpy()[:, n:] == 0.0)
            if k > 0:
                report["err_W"] = max(report["err_W"], rel_err(g["W"][b, h].numpy()[:k], o["W"][b, h, :k]))
            assert np.all(g["W"][b, h].numpy()[k:] == 0.0)
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
