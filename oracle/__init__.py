"""Plain fp64 CPU oracle for WildCat coreset attention — TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``wc_oracle.c`` (plain C, fp64, loops in the order the
method states them); this module compiles it with gcc on first use and wraps it
with ctypes.  ``forward`` runs the whole method over a batch of units:

    for each (batch b, kv head h):  unit = b * Hkv + h
        piv, F      = RPCholesky(K[b,h], r)          select
        W           = h(K_S,K_S)^-1 h(K_S,K) [V|1]   weights
        for each query head g of kv head h (GQA groups of Hq/Hkv):
            out[b,g] = rownorm(exp(beta Q K_S^T) W)  attend
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wc_oracle.c")
_LIB = os.path.join(_HERE, "libwc_oracle.so")
_lock = threading.Lock()
_lib = None

DEFAULT_EPS_STOP = 2.0 ** -20
REPLAY_WINDOW = 1e-6


def build(force: bool = False) -> str:
    """Compile wc_oracle.c into libwc_oracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "wc_oracle.h"))
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", _SRC, "-o", tmp, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB)
    return _LIB


class SelectInfo(ctypes.Structure):
    _fields_ = [
        ("rank", ctypes.c_int32),
        ("n_replays", ctypes.c_int32),
        ("failed_step", ctypes.c_int32),
        ("pad", ctypes.c_int32),
        ("max_margin", ctypes.c_double),
        ("fail_margin", ctypes.c_double),
    ]


def lib():
    """The oracle library (WC_ORACLE_LIB overrides the path; the mutation
    tests use it to load deliberately broken builds)."""
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(os.environ.get("WC_ORACLE_LIB") or build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            up = ctypes.POINTER(ctypes.c_uint32)
            L.wco_philox4x32_10.argtypes = [up, up, up]
            L.wco_philox4x32_10.restype = None
            L.wco_pivot_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32]
            L.wco_pivot_uniform.restype = ctypes.c_double
            L.wco_inverse_cdf.argtypes = [ctypes.c_int32, dp, ctypes.c_double]
            L.wco_inverse_cdf.restype = ctypes.c_int32
            L.wco_rpcholesky.argtypes = [
                ctypes.c_int32, ctypes.c_int32, dp, ctypes.c_double, ctypes.c_int32,
                ctypes.c_uint64, ctypes.c_uint32, ctypes.c_double,
                ip, ctypes.c_int32, ctypes.c_double,
                ip, dp, dp, dp, ctypes.POINTER(SelectInfo),
            ]
            L.wco_rpcholesky.restype = ctypes.c_int
            L.wco_nystrom_weights.argtypes = [
                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, dp, dp, ctypes.c_double,
                ctypes.c_int32, ip, dp,
            ]
            L.wco_nystrom_weights.restype = ctypes.c_int
            L.wco_coreset_values.argtypes = [
                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, dp, dp, ctypes.c_double,
                ctypes.c_int32, ip, dp,
            ]
            L.wco_coreset_values.restype = None
            L.wco_coreset_attend.argtypes = [
                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, dp, ctypes.c_int32, dp, dp,
                ctypes.c_double, dp,
            ]
            L.wco_coreset_attend.restype = None
            L.wco_exact_attention.argtypes = [
                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, dp, dp, dp,
                ctypes.c_double, dp,
            ]
            L.wco_exact_attention.restype = None
            _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    """Widen a torch tensor / array to a C-contiguous float64 numpy array."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch

        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def philox4x32_10(ctr, key) -> np.ndarray:
    c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
    o = (ctypes.c_uint32 * 4)()
    lib().wco_philox4x32_10(c, k, o)
    return np.array(list(o), dtype=np.uint32)


def pivot_uniform(seed: int, j: int, unit: int) -> float:
    return lib().wco_pivot_uniform(seed, j, unit)


def inverse_cdf(dg, t: float) -> int:
    a = _f64(dg)
    return int(lib().wco_inverse_cdf(len(a), _dp(a), t))


def default_beta(d: int) -> float:
    return 1.0 / np.sqrt(d)


def rpcholesky(K, r: int, beta: float, seed: int = 0, unit: int = 0,
               eps_stop: float = DEFAULT_EPS_STOP, replay_piv=None, replay_rank=None,
               window: float = REPLAY_WINDOW):
    """One unit.  Returns dict(piv, F (n x r), rank, dsum, dneg, info)."""
    K = _f64(K)
    n, d = K.shape
    piv = np.full(r, -1, dtype=np.int32)
    F = np.zeros((n, r), dtype=np.float64)
    dsum = np.zeros(r + 1, dtype=np.float64)
    dneg = np.zeros(1, dtype=np.float64)
    info = SelectInfo()
    rp = None
    rr = 0
    if replay_piv is not None:
        rp_arr = np.ascontiguousarray(np.asarray(replay_piv, dtype=np.int32))
        rp = _ip(rp_arr)
        rr = int(replay_rank if replay_rank is not None else int((rp_arr >= 0).sum()))
    rc = lib().wco_rpcholesky(n, d, _dp(K), beta, r, seed, unit, eps_stop, rp, rr, window,
                              _ip(piv), _dp(F), _dp(dsum), _dp(dneg), ctypes.byref(info))
    if rc != 0:
        raise ValueError("wco_rpcholesky: invalid arguments")
    return dict(piv=piv, F=F, rank=info.rank, dsum=dsum[: info.rank + 1], dneg=float(dneg[0]),
                n_replays=info.n_replays, failed_step=info.failed_step,
                max_margin=info.max_margin, fail_margin=info.fail_margin)


def coreset_values(K, V, piv, rank: int, beta: float) -> np.ndarray:
    K, V = _f64(K), _f64(V)
    n, d = K.shape
    dv = V.shape[1]
    p = np.ascontiguousarray(np.asarray(piv[:rank], dtype=np.int32))
    C1 = np.zeros((rank, dv + 1), dtype=np.float64)
    lib().wco_coreset_values(n, d, dv, _dp(K), _dp(V), beta, rank, _ip(p), _dp(C1))
    return C1


def nystrom_weights(K, V, piv, rank: int, beta: float) -> np.ndarray:
    K, V = _f64(K), _f64(V)
    n, d = K.shape
    dv = V.shape[1]
    p = np.ascontiguousarray(np.asarray(piv[:rank], dtype=np.int32))
    W = np.zeros((max(rank, 1), dv + 1), dtype=np.float64)
    rc = lib().wco_nystrom_weights(n, d, dv, _dp(K), _dp(V), beta, rank, _ip(p), _dp(W))
    if rc != 0:
        raise FloatingPointError("h(K_S, K_S) is numerically singular")
    return W[:rank]


def coreset_attend(Q, Ks, W, beta: float) -> np.ndarray:
    Q, Ks, W = _f64(Q), _f64(Ks), _f64(W)
    nq, d = Q.shape
    rank = Ks.shape[0]
    dv = W.shape[1] - 1
    out = np.zeros((nq, dv), dtype=np.float64)
    lib().wco_coreset_attend(nq, d, dv, _dp(Q), rank, _dp(Ks), _dp(W), beta, _dp(out))
    return out


def exact_attention(Q, K, V, beta: float) -> np.ndarray:
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    nq, d = Q.shape
    nk, dv = V.shape
    out = np.zeros((nq, dv), dtype=np.float64)
    lib().wco_exact_attention(nq, nk, d, dv, _dp(Q), _dp(K), _dp(V), beta, _dp(out))
    return out


def center_keys(K) -> np.ndarray:
    """Centring of one unit's keys, K - mean(K) over the keys, in fp64.
    [WildCat, gist.science summary, "Methodik" item 3: keys are re-centred by
    subtracting their mean; softmax attention is invariant to it.]"""
    K = _f64(K)
    return K - K.mean(axis=0, keepdims=True)


def forward(Q, K, V, r: int, seed: int = 0, beta: float | None = None,
            eps_stop: float = DEFAULT_EPS_STOP, replay=None, units=None, threads: int | None = None,
            bins: int = 1, center: bool = False):
    """Whole method over [B, Hq, nq, d] / [B, Hkv, n, d] / [B, Hkv, n, dv] inputs.

    replay: optional (piv [B, Hkv, r], rank [B, Hkv] (bins: [B, Hkv, bins]))
    decisions to replay (see wc_oracle.h).  units: optional list of unit
    indices to compute (the others are left as zeros / -1).

    bins > 1 (the pages' divide-and-conquer selection, "Methodik" item 1,
    "Effizienz"; the bin layout and per-bin weights are this build's reading):
    each unit's keys split into `bins` contiguous bins of n / bins keys; bin b
    runs RPCholesky with r / bins pivots on its keys (Philox unit index
    u * bins + b) and Nystrom weights on its keys and values; attention runs over
    the union of the bins' coresets.  F is then [B, Hkv, n, r] block diagonal
    (bin b's keys x bin b's columns).

    center: the selection and the weights use K - mean(K) per unit; attention
    uses the centred coreset keys too (equal to the raw keys' result, by the
    invariance).  Returns a dict of numpy arrays.
    """
    Qa, Ka, Va = _f64(Q), _f64(K), _f64(V)
    B, Hq, nq, d = Qa.shape
    _, Hkv, n, _ = Ka.shape
    dv = Va.shape[-1]
    if beta is None:
        beta = default_beta(d)
    nb = max(int(bins), 1)
    if n % nb or r % nb:
        raise ValueError("n and r must be multiples of bins")
    nbk, rb = n // nb, r // nb
    group = Hq // Hkv
    nunits = B * Hkv
    piv = np.full((B, Hkv, r), -1, dtype=np.int32)
    rank = np.zeros((B, Hkv, nb), dtype=np.int32)
    F = np.zeros((B, Hkv, n, r), dtype=np.float64)
    W = np.zeros((B, Hkv, r, dv + 1), dtype=np.float64)
    out = np.zeros((B, Hq, nq, dv), dtype=np.float64)
    infos = [None] * (nunits * nb)
    todo = list(range(nunits)) if units is None else list(units)

    def run(u):
        b, h = divmod(u, Hkv)
        Ku = center_keys(Ka[b, h]) if center else Ka[b, h]
        rows = []
        for bb in range(nb):
            ks, ke = bb * nbk, (bb + 1) * nbk
            rp = rr = None
            if replay is not None:
                rp = np.asarray(replay[0])[b, h, bb * rb:(bb + 1) * rb].copy()
                rp[rp >= 0] -= ks
                rr_all = np.asarray(replay[1])
                rr = int(rr_all[b, h, bb] if rr_all.ndim == 3 else rr_all[b, h])
            res = rpcholesky(Ku[ks:ke], rb, beta, seed=seed, unit=u * nb + bb, eps_stop=eps_stop,
                             replay_piv=rp, replay_rank=rr)
            k = res["rank"]
            pb = res["piv"].copy()
            pb[pb >= 0] += ks
            piv[b, h, bb * rb:(bb + 1) * rb] = pb
            rank[b, h, bb] = k
            F[b, h, ks:ke, bb * rb:(bb + 1) * rb] = res["F"]
            infos[u * nb + bb] = res
            if k > 0:
                W[b, h, bb * rb:bb * rb + k] = nystrom_weights(Ku[ks:ke], Va[b, h, ks:ke], res["piv"], k, beta)
                rows.extend(range(bb * rb, bb * rb + k))
        if rows:
            sel = piv[b, h, rows]
            Ks = Ku[sel]
            for g in range(group):
                out[b, h * group + g] = coreset_attend(Qa[b, h * group + g], Ks, W[b, h, rows], beta)
        else:
            out[b, h * group:(h + 1) * group] = np.nan

    nthreads = threads or min(len(todo), os.cpu_count() or 1)
    if nthreads <= 1 or len(todo) <= 1:
        for u in todo:
            run(u)
    else:
        with ThreadPoolExecutor(max_workers=nthreads) as ex:
            list(ex.map(run, todo))
    if nb == 1:
        rank = rank[..., 0]
    return dict(piv=piv, rank=rank, F=F, W=W, out=out, info=infos, beta=beta)
