"""Seeded synthetic inputs for the WildCat workloads.

This module holds no arithmetic of the method: it only draws Q, K, V with the
shapes, value distributions and structure of the workloads below, so that the
CUDA path and the CPU oracle can be fed the same values.  Every draw is made in
fp64 on a CPU ``torch.Generator`` seeded with ``seed``, in the order Q, K, V,
then clipped and cast to the storage dtype.

Workloads (batch x kv-heads, n keys, d = dv, coreset size r):

* ``tiny``     1 head, n = nq = 512, d = 64, r = 32, fp32; rows N(0, I) scaled
               to norm <= 4 (bounded inputs).
* ``vit``      64 x 12 heads, n = nq = 1024 (32 x 32 patches), d = 64, r = 64,
               bf16; rows N(0, I) clipped to norm <= 8.  Stands in for the
               image-classification experiment (only its shape).
* ``diffusion`` 2 x 16 heads, n = nq = 4096 (64 x 64 latent), d = 64, r = 256,
               bf16; keys from a 32-centre Gaussian mixture (centres N(0, I),
               within-cluster sigma 0.3), queries and values N(0, I).
* ``kv``       1 batch, 32 query heads over 8 kv heads (GQA), 32768 keys,
               256 decode queries, d = 128, r = 1024, bf16; rows N(0, I)
               clipped to norm <= 12.  Stands in for the KV-cache compression
               experiment (only its shape).
* ``long``     1 x 8 heads, n = nq = 131072, d = 128, r = 2048, bf16; 95 % of
               keys from a 256-centre mixture (centres N(0, I), sigma 0.3), 5 %
               uniform outliers with coordinates iid U[-sqrt 3, sqrt 3] at a
               random 5 % of positions; queries and values N(0, I).
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    n_k: int
    n_q: int
    d: int
    dv: int
    r: int
    dtype: str            # "f32" or "bf16"
    keys: str             # "gauss" or "mixture"
    clip: float | None    # row-norm bound, None for unclipped
    centres: int = 0
    sigma: float = 0.0
    outlier_frac: float = 0.0

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 512, 512, 64, 64, 32, "f32", "gauss", 4.0),
    "vit": Workload("vit", 64, 12, 12, 1024, 1024, 64, 64, 64, "bf16", "gauss", 8.0),
    "diffusion": Workload("diffusion", 2, 16, 16, 4096, 4096, 64, 64, 256, "bf16", "mixture", None,
                          centres=32, sigma=0.3),
    "kv": Workload("kv", 1, 32, 8, 32768, 256, 128, 128, 1024, "bf16", "gauss", 12.0),
    "long": Workload("long", 1, 8, 8, 131072, 131072, 128, 128, 2048, "bf16", "mixture", None,
                     centres=256, sigma=0.3, outlier_frac=0.05),
}


def _clip_rows(x: torch.Tensor, bound: float | None) -> torch.Tensor:
    if bound is None:
        return x
    norm = x.norm(dim=-1, keepdim=True)
    return x * torch.clamp(bound / norm.clamp_min(1e-300), max=1.0)


def _keys(w: Workload, g: torch.Generator) -> torch.Tensor:
    units = w.batch * w.hkv
    if w.keys == "gauss":
        return torch.randn(units, w.n_k, w.d, generator=g, dtype=torch.float64)
    centres = torch.randn(units, w.centres, w.d, generator=g, dtype=torch.float64)
    z = torch.randint(0, w.centres, (units, w.n_k), generator=g)
    noise = torch.randn(units, w.n_k, w.d, generator=g, dtype=torch.float64)
    k = torch.gather(centres, 1, z.unsqueeze(-1).expand(-1, -1, w.d)) + w.sigma * noise
    if w.outlier_frac > 0.0:
        n_out = int(round(w.outlier_frac * w.n_k))
        a = math.sqrt(3.0)
        for u in range(units):
            pos = torch.randperm(w.n_k, generator=g)[:n_out]
            vals = (torch.rand(n_out, w.d, generator=g, dtype=torch.float64) * 2.0 - 1.0) * a
            k[u, pos] = vals
    return k


def make_inputs(w: Workload, seed: int = 0):
    """Return (Q, K, V) as contiguous CPU tensors in the workload's dtype.

    Shapes: Q [B, Hq, n_q, d], K [B, Hkv, n_k, d], V [B, Hkv, n_k, dv].
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(w.batch * w.hq, w.n_q, w.d, generator=g, dtype=torch.float64)
    k = _keys(w, g)
    v = torch.randn(w.batch * w.hkv, w.n_k, w.dv, generator=g, dtype=torch.float64)
    if w.clip is not None:
        q, k, v = _clip_rows(q, w.clip), _clip_rows(k, w.clip), _clip_rows(v, w.clip)
    dt = w.torch_dtype
    q = q.reshape(w.batch, w.hq, w.n_q, w.d).to(dt).contiguous()
    k = k.reshape(w.batch, w.hkv, w.n_k, w.d).to(dt).contiguous()
    v = v.reshape(w.batch, w.hkv, w.n_k, w.dv).to(dt).contiguous()
    return q, k, v
