"""Python binding of the WildCat C ABI (include/wildcat.h).

Argument marshalling only: every step runs in libwildcat.so's CUDA kernels.
Tensors are torch CUDA tensors (PyTorch supplies device memory and streams);
the functions raise if the library is missing or a call fails.

    from coreset_attention_approximation_b200 import wildcat
    res = wildcat.forward(Q, K, V, r=64, seed=0)        # dict with out, piv, rank, F, Ks, W
"""

from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwildcat.so")

WC_F32, WC_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "CUDA error", 3: "device-side wait timed out",
          4: "unsupported shape", 5: "workspace too small", 6: "non-finite value on the device",
          7: "index outside its buffer (debug build)"}


class WildcatError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)} ({code})")
        self.code = code


class WcShape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("hq", ctypes.c_int32), ("hkv", ctypes.c_int32),
        ("n_k", ctypes.c_int32), ("n_q", ctypes.c_int32), ("d", ctypes.c_int32),
        ("dv", ctypes.c_int32), ("r", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("scale", ctypes.c_float), ("eps_stop", ctypes.c_float), ("wait_timeout_ms", ctypes.c_uint32),
        ("seed", ctypes.c_uint64), ("bins", ctypes.c_int32), ("center", ctypes.c_int32),
        ("unit_base", ctypes.c_int32),
    ]


EXPORTS = [
    "wc_f_ld", "wc_workspace_bytes", "wc_forward_workspace_bytes", "wc_select", "wc_weights", "wc_attend",
    "wc_forward", "wc_check_device_status", "wc_selftest_wait_timeout", "wc_status_string",
    "wc_attend_noalloc", "wc_selftest_exp2", "wc_read_bandwidth_probe",
]

_lib = None


def use_debug_library(debug: bool = True) -> None:
    """Switch to the bounds-checked build (libwildcat_debug.so, built by
    `python -m coreset_attention_approximation_b200.build --debug`): its kernels
    check every data-dependent index (pivots, ranks) against its buffer and
    record WC_ERR_BOUNDS instead of making the access.  Takes effect for calls
    made after it."""
    global LIB_PATH, _lib
    LIB_PATH = os.path.join(HERE, "libwildcat_debug.so" if debug else "libwildcat.so")
    _lib = None


def lib():
    """Load libwildcat.so (built by `python -m coreset_attention_approximation_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m coreset_attention_approximation_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(WcShape)
        L.wc_f_ld.argtypes, L.wc_f_ld.restype = [ctypes.c_int32], ctypes.c_int64
        L.wc_workspace_bytes.argtypes, L.wc_workspace_bytes.restype = [sp], sz
        L.wc_forward_workspace_bytes.argtypes, L.wc_forward_workspace_bytes.restype = [sp], sz
        L.wc_select.argtypes, L.wc_select.restype = [sp, vp, vp, vp, vp, vp, sz, vp], i32
        L.wc_weights.argtypes, L.wc_weights.restype = [sp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i32
        L.wc_attend.argtypes, L.wc_attend.restype = [sp, vp, vp, vp, vp, vp, vp, sz, vp], i32
        L.wc_forward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.wc_forward.restype = i32
        L.wc_check_device_status.argtypes, L.wc_check_device_status.restype = [vp, vp], i32
        L.wc_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, vp]
        L.wc_selftest_wait_timeout.restype = i32
        L.wc_status_string.argtypes, L.wc_status_string.restype = [i32], ctypes.c_char_p
        L.wc_attend_noalloc.argtypes, L.wc_attend_noalloc.restype = [sp, vp, vp, vp, vp, vp, vp], i32
        L.wc_selftest_exp2.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int32, vp]
        L.wc_selftest_exp2.restype = i32
        L.wc_read_bandwidth_probe.argtypes = [vp, ctypes.c_int64, vp, vp]
        L.wc_read_bandwidth_probe.restype = i32
        _lib = L
    return _lib


def _check(code: int, what: str):
    if code != 0:
        raise WildcatError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_shape(batch, hq, hkv, n_k, n_q, d, dv, r, dtype, scale=0.0, eps_stop=0.0, seed=0,
               wait_timeout_ms=0, bins=1, center=False, unit_base=0) -> WcShape:
    code = {torch.float32: WC_F32, torch.bfloat16: WC_BF16}.get(dtype, dtype)
    return WcShape(batch, hq, hkv, n_k, n_q, d, dv, r, code, scale, eps_stop, wait_timeout_ms, seed,
                   int(bins), int(bool(center)), int(unit_base))


def shape_of(Q, K, V, r, **kw) -> WcShape:
    B, Hkv, n, d = K.shape
    dv = V.shape[-1]
    if Q is None:
        Hq, nq = Hkv, 0
    else:
        Hq, nq = Q.shape[1], Q.shape[2]
    return make_shape(B, Hq, Hkv, n, nq, d, dv, r, K.dtype, **kw)


def f_ld(n_k: int) -> int:
    return int(lib().wc_f_ld(n_k))


def workspace_bytes(shape: WcShape) -> int:
    return int(lib().wc_workspace_bytes(ctypes.byref(shape)))


def forward_workspace_bytes(shape: WcShape) -> int:
    return int(lib().wc_forward_workspace_bytes(ctypes.byref(shape)))


def workspace(shape: WcShape, device, forward_room: bool = False) -> torch.Tensor:
    n = forward_workspace_bytes(shape) if forward_room else workspace_bytes(shape)
    if n == 0:
        raise WildcatError(1, "workspace size")
    # the device status word at offset 0 starts clear
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _outputs(shape: WcShape, device, dtype):
    B, Hkv, r, n = shape.batch, shape.hkv, shape.r, shape.n_k
    nb = max(shape.bins, 1)
    if nb > 1:
        # bins: per-bin ranks and per-bin factors over each bin's keys
        rank = torch.empty(B, Hkv, nb, dtype=torch.int32, device=device)
        F = torch.empty(B, Hkv, nb, r // nb, f_ld(n // nb), dtype=torch.float32, device=device)
    else:
        rank = torch.empty(B, Hkv, dtype=torch.int32, device=device)
        F = torch.empty(B, Hkv, r, f_ld(n), dtype=torch.float32, device=device)
    return dict(
        piv=torch.empty(B, Hkv, r, dtype=torch.int32, device=device),
        rank=rank,
        F=F,
        Ks=torch.empty(B, Hkv, r, shape.d, dtype=dtype, device=device),
        W=torch.empty(B, Hkv, r, shape.dv + 1, dtype=torch.float32, device=device),
    )


def select(K, r, seed=0, *, ws=None, stream=None, **kw):
    shape = shape_of(None, K, K[..., :8], r, seed=seed, **kw)
    o = _outputs(shape, K.device, K.dtype)
    ws = workspace(shape, K.device) if ws is None else ws
    _check(lib().wc_select(ctypes.byref(shape), _ptr(K), _ptr(o["piv"]), _ptr(o["F"]), _ptr(o["rank"]),
                           _ptr(ws), ws.numel(), _stream(stream)), "wc_select")
    return dict(piv=o["piv"], F=o["F"], rank=o["rank"], ws=ws)


def weights(K, V, piv, F, rank, r, *, ws=None, stream=None, **kw):
    shape = shape_of(None, K, V, r, **kw)
    o = _outputs(shape, K.device, K.dtype)
    ws = workspace(shape, K.device) if ws is None else ws
    _check(lib().wc_weights(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(piv), _ptr(F), _ptr(rank),
                            _ptr(o["Ks"]), _ptr(o["W"]), _ptr(ws), ws.numel(), _stream(stream)), "wc_weights")
    return dict(Ks=o["Ks"], W=o["W"], ws=ws)


def attend(Q, Ks, W, rank, n_k, *, ws=None, stream=None, **kw):
    B, Hq, nq, d = Q.shape
    Hkv, r, dv = Ks.shape[1], Ks.shape[2], W.shape[-1] - 1
    shape = make_shape(B, Hq, Hkv, n_k, nq, d, dv, r, Q.dtype, **kw)
    out = torch.empty(B, Hq, nq, dv, dtype=torch.float32, device=Q.device)
    ws = workspace(shape, Q.device) if ws is None else ws
    _check(lib().wc_attend(ctypes.byref(shape), _ptr(Q), _ptr(Ks), _ptr(W), _ptr(rank), _ptr(out),
                           _ptr(ws), ws.numel(), _stream(stream)), "wc_attend")
    return out


def attend_noalloc(Q, Ks, W, rank, n_k, *, out=None, stream=None, **kw):
    """wc_attend_noalloc: attention with the library's fixed device scratch,
    for callers that cannot allocate.  `out` may be preallocated."""
    B, Hq, nq, d = Q.shape
    Hkv, r, dv = Ks.shape[1], Ks.shape[2], W.shape[-1] - 1
    shape = make_shape(B, Hq, Hkv, n_k, nq, d, dv, r, Q.dtype, **kw)
    if out is None:
        out = torch.empty(B, Hq, nq, dv, dtype=torch.float32, device=Q.device)
    _check(lib().wc_attend_noalloc(ctypes.byref(shape), _ptr(Q), _ptr(Ks), _ptr(W), _ptr(rank), _ptr(out),
                                   _stream(stream)), "wc_attend_noalloc")
    return out


def forward(Q, K, V, r, seed=0, *, ws=None, stream=None, outputs=None, **kw):
    """Whole path on the GPU: select -> weights -> attend.

    Q [B,Hq,nq,d], K [B,Hkv,n,d], V [B,Hkv,n,dv] CUDA tensors (bf16 or fp32,
    contiguous).  `outputs` may hold preallocated tensors (out, piv, rank, F,
    Ks, W); missing ones are allocated.  Returns the dict of all of them.
    """
    shape = shape_of(Q, K, V, r, seed=seed, **kw)
    o = dict(outputs or {})
    if any(k not in o for k in ("piv", "rank", "F", "Ks", "W")):
        for k, v in _outputs(shape, K.device, K.dtype).items():
            o.setdefault(k, v)
    o.setdefault("out", torch.empty(Q.shape[0], Q.shape[1], Q.shape[2], shape.dv, dtype=torch.float32,
                                    device=K.device))
    ws = workspace(shape, K.device) if ws is None else ws
    _check(lib().wc_forward(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(o["out"]), _ptr(o["piv"]),
                            _ptr(o["rank"]), _ptr(o["F"]), _ptr(o["Ks"]), _ptr(o["W"]), _ptr(ws), ws.numel(),
                            _stream(stream)), "wc_forward")
    o["ws"] = ws
    return o


class ForwardGraph:
    """wc_forward captured once into a CUDA graph, then replayed: repeated
    forward passes over the same device buffers cost one graph launch instead
    of the path's kernel launches and memsets.  Refill Q, K, V in place (for
    example with copy_) before each `replay()`; the outputs (out, piv, rank, F,
    Ks, W) are overwritten in place and returned."""

    def __init__(self, Q, K, V, r, seed=0, *, ws=None, outputs=None, **kw):
        self.Q, self.K, self.V = Q, K, V
        self.shape = shape_of(Q, K, V, r, seed=seed, **kw)
        self.ws = workspace(self.shape, K.device) if ws is None else ws
        o = dict(outputs or {})
        if any(k not in o for k in ("piv", "rank", "F", "Ks", "W")):
            for k, v in _outputs(self.shape, K.device, K.dtype).items():
                o.setdefault(k, v)
        o.setdefault("out", torch.empty(Q.shape[0], Q.shape[1], Q.shape[2], self.shape.dv, dtype=torch.float32,
                                        device=K.device))
        self.outputs = o
        # one eager pass first: function attributes and tensor maps are set up outside the capture
        self._launch(torch.cuda.current_stream(K.device))
        torch.cuda.current_stream(K.device).synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._launch(torch.cuda.current_stream(K.device))

    def _launch(self, stream):
        o = self.outputs
        _check(lib().wc_forward(ctypes.byref(self.shape), _ptr(self.Q), _ptr(self.K), _ptr(self.V), _ptr(o["out"]),
                                _ptr(o["piv"]), _ptr(o["rank"]), _ptr(o["F"]), _ptr(o["Ks"]), _ptr(o["W"]),
                                _ptr(self.ws), self.ws.numel(), _stream(stream)), "wc_forward")

    def replay(self):
        self.graph.replay()
        return self.outputs


class HostPipeline:
    """Forward passes over a sequence of host batches, with the copies
    overlapped: batch i+1's host-to-device copy and batch i-1's device-to-host
    copy run on their own streams while batch i computes.  Two device copies
    of Q, K, V and out alternate; the factor, weights and workspace are shared
    (the passes themselves run one after another on the compute stream).

    Host tensors must be pinned for the copies to overlap.  Every batch has
    the shapes and dtype of the (Q, K, V) given here."""

    def __init__(self, Q, K, V, r, seed=0, *, device="cuda", stream=None, ws=None, outputs=None, **kw):
        """Q, K, V: host tensors of the batches' shapes and dtype (only their
        shapes are read).  ws / outputs: optional workspace and (piv, rank, F,
        Ks, W) device tensors to reuse; the last batch's stay there."""
        self.device = torch.device(device)
        self.r, self.seed, self.kw = r, seed, kw
        self.shape = shape_of(Q, K, V, r, seed=seed, **kw)
        self.ws = workspace(self.shape, self.device) if ws is None else ws
        self.shared = {k: v for k, v in (outputs or {}).items() if k != "out"}
        if any(k not in self.shared for k in ("piv", "rank", "F", "Ks", "W")):
            for k, v in _outputs(self.shape, self.device, K.dtype).items():
                self.shared.setdefault(k, v)
        out_shape = (Q.shape[0], Q.shape[1], Q.shape[2], self.shape.dv)
        self.bufs = [dict(Q=torch.empty(Q.shape, dtype=Q.dtype, device=self.device),
                          K=torch.empty(K.shape, dtype=K.dtype, device=self.device),
                          V=torch.empty(V.shape, dtype=V.dtype, device=self.device),
                          out=torch.empty(out_shape, dtype=torch.float32, device=self.device)) for _ in range(2)]
        self.compute = stream or torch.cuda.current_stream(self.device)
        self.h2d = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.loaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.drained = [torch.cuda.Event() for _ in range(2)]
        self.started = [False, False]

    def run(self, batches):
        """batches: iterable of (Q, K, V, out) host tensors; out [B, Hq, nq, dv]
        fp32 receives the batch's output.  The copies and passes are queued
        behind whatever the compute stream already holds; returns once the
        last output has been queued (call `wait()` before reading it)."""
        for i, (Qh, Kh, Vh, oh) in enumerate(batches):
            j = i % 2
            b = self.bufs[j]
            with torch.cuda.stream(self.h2d):
                if i == 0:
                    self.h2d.wait_stream(self.compute)            # after whatever the caller queued
                if self.started[j]:
                    self.h2d.wait_event(self.computed[j])     # batch i-2 has finished reading buffer j
                b["Q"].copy_(Qh, non_blocking=True)
                b["K"].copy_(Kh, non_blocking=True)
                b["V"].copy_(Vh, non_blocking=True)
                self.loaded[j].record(self.h2d)
            self.compute.wait_event(self.loaded[j])
            if self.started[j]:
                self.compute.wait_event(self.drained[j])       # batch i-2's output has left buffer j
            forward(b["Q"], b["K"], b["V"], self.r, self.seed, ws=self.ws, stream=self.compute,
                    outputs=dict(self.shared, out=b["out"]), **self.kw)
            self.computed[j].record(self.compute)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(self.computed[j])
                oh.copy_(b["out"], non_blocking=True)
                self.drained[j].record(self.d2h)
            self.started[j] = True
        # the compute stream ends after the last copy out
        self.compute.wait_stream(self.d2h)

    def wait(self):
        self.compute.synchronize()
        return check_device_status(self.ws, self.compute)


def check_device_status(ws, stream=None) -> int:
    return int(lib().wc_check_device_status(_ptr(ws), _stream(stream)))


def selftest_wait_timeout(ws, timeout_ms, stream=None) -> int:
    return int(lib().wc_selftest_wait_timeout(_ptr(ws), ws.numel(), timeout_ms, _stream(stream)))


def read_probe(buf, sink, stream=None):
    """Reads the CUDA tensor `buf` once as a read-only stream (the read
    bandwidth probe); `sink` (one int32 on the device) receives the XOR of its
    32-bit words."""
    _check(lib().wc_read_bandwidth_probe(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink), _stream(stream)),
           "wc_read_bandwidth_probe")


def selftest_exp2(x, method=0, stream=None):
    """2^x for an fp32 CUDA tensor as the tensor-core kernels compute it:
    method 0 on the FMA / ALU pipes (the polynomial), 1 on the exponential unit."""
    y = torch.empty_like(x)
    _check(lib().wc_selftest_exp2(_ptr(x), _ptr(y), x.numel(), method, _stream(stream)), "wc_selftest_exp2")
    return y
