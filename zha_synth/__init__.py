"""Seeded synthetic inputs for the ZHA hot path.

This module is shared by the CPU oracle (``oracle/``), the GPU tests and the
benchmark.  It holds no arithmetic of the method itself: it only draws keys,
values, queries and reference queries with the shapes and value distributions
of the long-context decode / prefill workloads, so that both sides of a parity
test see the very same bytes.

Recipe (one independent draw per (batch, KV head) unit):
  * centres   c_j ~ N(0, I_d),                       j < n_centres
  * keys      k_t = c_{z_t} + 0.3 * N(0, I_d),        z_t ~ U{0..n_centres-1} i.i.d.
  * values    v_t ~ N(0, I_d)
  * queries   q   = 2 * c_{z'} + 0.3 * N(0, I_d)      z' ~ U over the query's KV group
              (a fraction ``random_frac`` of queries instead use q = 2 * N(0, I_d))
  * reference queries  q_hat_r ~ N(0, I_d / d)        (randomly initialised, never trained)
With ``segment`` > 0 (a structured variant, not one of the five workloads) the cluster of a
key is drawn once per run of ``segment`` consecutive positions instead of per key, and a
query takes the centre of a uniformly chosen segment of its cache: the keys that matter to a
query then sit in a few contiguous chunks, as in text where a topic spans a passage.
Keys, values and queries are drawn in fp32 and then stored in the workload's
dtype (bf16 rounding is round-to-nearest-even, torch's ``.to(torch.bfloat16)``).

Every stream of random numbers has its own generator seeded from
``(seed, stream tag)``, so a component's values do not depend on the sizes of
the other components.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

__all__ = [
    "Workload", "WORKLOADS", "workload", "scaled",
    "clustered_kv", "queries", "reference_queries", "new_tokens", "segment_centres",
]

_TAGS = {"centres": 11, "assign": 12, "knoise": 13, "values": 14, "qpick": 21,
         "qnoise": 22, "qrand": 23, "qmix": 24, "qref": 31, "new_assign": 41,
         "new_knoise": 42, "new_values": 43}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: geometry, tree shape, threshold and generator."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int                 # keys already in the cache
    n_centres: int
    depth: int             # summary levels L
    p: tuple               # routing thresholds to run
    R: int = 4             # reference queries per KV head
    leaf: int = 64
    branch: int = 16
    dtype: str = "bf16"    # "bf16" or "f32" (K, V, Q, O)
    seed: int = 0
    mode: str = "decode"   # "decode": one new token per sequence; "prefill": n_new causal tokens
    n_new: int = 1
    random_frac: float = 0.0
    segment: int = 0       # > 0: keys share a centre over runs of this many positions

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def t_cap(self) -> int:
        """Cache capacity: the existing keys plus the appended ones, rounded up to a
        whole leaf chunk."""
        n = self.T + self.n_new
        return (n + self.leaf - 1) // self.leaf * self.leaf


# The five workloads of the long-context study.  Reference-query count R=4 for
# all of them; where a centre count is not stated, 4096 is used.
WORKLOADS = {
    "tiny-decode-f32": Workload("tiny-decode-f32", B=1, Hq=4, Hkv=1, d=128, T=8192,
                                n_centres=256, depth=2, p=(0.9,), dtype="f32", seed=0),
    "batched-decode-128k": Workload("batched-decode-128k", B=32, Hq=32, Hkv=4, d=128,
                                    T=131072, n_centres=4096, depth=3, p=(0.95,), seed=1),
    "prefill-append-256k": Workload("prefill-append-256k", B=1, Hq=16, Hkv=2, d=128,
                                    T=262144, n_centres=4096, depth=4, p=(0.95,), seed=2,
                                    mode="prefill", n_new=4096, random_frac=0.1),
    "long-decode-1m": Workload("long-decode-1m", B=4, Hq=32, Hkv=4, d=128, T=1048576,
                               n_centres=4096, depth=5, p=(0.95, 0.99), seed=3),
    "deep-tree-16m": Workload("deep-tree-16m", B=1, Hq=8, Hkv=1, d=128, T=16777216,
                              n_centres=65536, depth=6, p=(0.95,), seed=4),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(w: Workload, T: int, B: Optional[int] = None, n_new: Optional[int] = None,
           n_centres: Optional[int] = None) -> Workload:
    """Same generator and geometry with a smaller cache (and optionally batch)."""
    kw = dict(T=T, name=f"{w.name}@T{T}")
    if B is not None:
        kw["B"] = B
    if n_new is not None:
        kw["n_new"] = n_new
    if n_centres is not None:
        kw["n_centres"] = n_centres
    return dataclasses.replace(w, **kw)


def _gen(device, seed: int, tag: str, sub: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + _TAGS[tag] * 7919 + sub * 104729) % (2**63 - 1))
    return g


def _tdtype(dtype: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]


def centres_of(w: Workload, device="cpu") -> torch.Tensor:
    """Cluster centres, [B, Hkv, n_centres, d] fp32."""
    g = _gen(device, w.seed, "centres")
    return torch.randn(w.B, w.Hkv, w.n_centres, w.d, generator=g, device=device)


def segment_centres(w: Workload, b: int, h: int, device="cpu") -> torch.Tensor:
    """Centre index of every run of ``w.segment`` positions of unit (b, h), over t_cap."""
    ga = _gen(device, w.seed, "assign", b * w.Hkv + h)
    nseg = (w.t_cap + w.segment - 1) // w.segment
    return torch.randint(0, w.n_centres, (nseg,), generator=ga, device=device)


def clustered_kv(w: Workload, device="cpu", block: int = 1 << 20):
    """Keys/values for the existing cache, laid out [B, Hkv, t_cap, d].

    Positions >= T are zero (they are filled by the appended tokens).  The draw
    is done in blocks of ``block`` positions per (b, h) unit to bound the
    temporary fp32 memory.  Returns (centres, K, V).
    """
    C = centres_of(w, device)
    dt = _tdtype(w.dtype)
    K = torch.zeros(w.B, w.Hkv, w.t_cap, w.d, dtype=dt, device=device)
    V = torch.zeros_like(K)
    for b in range(w.B):
        for h in range(w.Hkv):
            unit = b * w.Hkv + h
            ga = _gen(device, w.seed, "assign", unit)
            gk = _gen(device, w.seed, "knoise", unit)
            gv = _gen(device, w.seed, "values", unit)
            zs = segment_centres(w, b, h, device) if w.segment > 0 else None
            for t0 in range(0, w.T, block):
                n = min(block, w.T - t0)
                if zs is not None:
                    z = zs[(t0 + torch.arange(n, device=device)) // w.segment]
                else:
                    z = torch.randint(0, w.n_centres, (n,), generator=ga, device=device)
                k = C[b, h][z] + 0.3 * torch.randn(n, w.d, generator=gk, device=device)
                K[b, h, t0:t0 + n] = k.to(dt)
                V[b, h, t0:t0 + n] = torch.randn(n, w.d, generator=gv, device=device).to(dt)
    return C, K, V


def new_tokens(w: Workload, C: torch.Tensor, n_new: int, device="cpu", step: int = 0):
    """Keys/values of ``n_new`` appended tokens, [B, n_new, Hkv, d] (model layout)."""
    dt = _tdtype(w.dtype)
    ga = _gen(device, w.seed, "new_assign", step)
    gk = _gen(device, w.seed, "new_knoise", step)
    gv = _gen(device, w.seed, "new_values", step)
    z = torch.randint(0, w.n_centres, (w.B, n_new, w.Hkv), generator=ga, device=device)
    if w.segment > 0:                                # the runs continue past T
        pos = (w.T + step * n_new + torch.arange(n_new, device=device)) // w.segment
        for b in range(w.B):
            for h in range(w.Hkv):
                zs = segment_centres(w, b, h, device)
                z[b, :, h] = zs[pos.clamp(max=len(zs) - 1)]
    bi = torch.arange(w.B, device=device).view(-1, 1, 1)
    hi = torch.arange(w.Hkv, device=device).view(1, 1, -1)
    k = C[bi, hi, z] + 0.3 * torch.randn(w.B, n_new, w.Hkv, w.d, generator=gk, device=device)
    v = torch.randn(w.B, n_new, w.Hkv, w.d, generator=gv, device=device)
    return k.to(dt), v.to(dt)


def queries(w: Workload, C: torch.Tensor, nq: int, device="cpu", step: int = 0):
    """Queries [B, nq, Hq, d] near the centres of each head's KV group.

    A fraction ``w.random_frac`` of (query, head) pairs, chosen i.i.d., are
    isotropic Gaussian directions 2*N(0, I) instead.
    """
    dt = _tdtype(w.dtype)
    gp = _gen(device, w.seed, "qpick", step)
    gn = _gen(device, w.seed, "qnoise", step)
    z = torch.randint(0, w.n_centres, (w.B, nq, w.Hq), generator=gp, device=device)
    if w.segment > 0:                                # the centre of a random full segment
        nfull = max(1, w.T // w.segment)
        pick = torch.randint(0, nfull, (w.B, nq, w.Hq), generator=gp, device=device)
        for b in range(w.B):
            for h in range(w.Hkv):
                zs = segment_centres(w, b, h, device)
                z[b, :, h * w.G:(h + 1) * w.G] = zs[pick[b, :, h * w.G:(h + 1) * w.G]]
    bi = torch.arange(w.B, device=device).view(-1, 1, 1)
    gi = (torch.arange(w.Hq, device=device) // w.G).view(1, 1, -1)
    q = 2.0 * C[bi, gi, z] + 0.3 * torch.randn(w.B, nq, w.Hq, w.d, generator=gn, device=device)
    if w.random_frac > 0:
        gr = _gen(device, w.seed, "qrand", step)
        gm = _gen(device, w.seed, "qmix", step)
        rnd = 2.0 * torch.randn(w.B, nq, w.Hq, w.d, generator=gr, device=device)
        mix = torch.rand(w.B, nq, w.Hq, generator=gm, device=device) < w.random_frac
        q = torch.where(mix[..., None], rnd, q)
    return q.to(dt)


def reference_queries(w: Workload, device="cpu") -> torch.Tensor:
    """Randomly initialised reference queries, [Hkv, R, d] fp32, N(0, I/d)."""
    g = _gen(device, w.seed, "qref")
    return torch.randn(w.Hkv, w.R, w.d, generator=g, device=device) / (w.d ** 0.5)
