"""Shared harness of the GPU parity tests: seeded inputs on the device, the library
through its C ABI, and the CPU oracle on the same bytes (copied to the host)."""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

import zha_synth as S
from oracle import zha_oracle as zo

NEAR_CUTOFF = 1e-4      # cumulative-probability margin below which a cutoff is "near"


def geometry(w: S.Workload, t_cap: Optional[int] = None):
    import hierarchical_sparse_attention_02_b200 as Z
    return Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=t_cap or w.t_cap, depth=w.depth, R=w.R,
                      d=w.d, leaf=w.leaf, branch=w.branch,
                      dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)


def route_storage(w: S.Workload) -> str:
    return "bf16" if w.dtype == "bf16" else "f32"


def tree_arrays(g, tree: torch.Tensor, level: int):
    """Views of one level of the device tree buffer: (k_route, b_hat, F, k_state)."""
    import hierarchical_sparse_attention_02_b200 as Z
    L = Z.tree_level(g, level)
    n = g.B * g.Hkv * L.n_cap
    es = 2 if g.dtype == torch.bfloat16 else 4
    kr = tree[L.k_route_off:L.k_route_off + n * g.R * g.d * es].view(g.dtype).view(g.B, g.Hkv, L.n_cap, g.R, g.d)
    bh = tree[L.b_hat_off:L.b_hat_off + n * g.R * 4].view(torch.float32).view(g.B, g.Hkv, L.n_cap, g.R)
    F = tree[L.F_off:L.F_off + n * g.R * 4].view(torch.float32).view(g.B, g.Hkv, L.n_cap, g.R)
    ks = tree[L.k_state_off:L.k_state_off + n * g.R * g.d * 4].view(torch.float32).view(g.B, g.Hkv, L.n_cap, g.R, g.d)
    return kr, bh, F, ks


def bf16_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place between two arrays of bf16 values."""
    def ordinal(x):
        bits = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16)
        v = bits.to(torch.int64).numpy()
        v = np.where(v < 0, -(v & 0x7FFF), v)
        return v
    return np.abs(ordinal(a) - ordinal(b))


def f32_ulp_diff(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    def ordinal(x):
        v = np.ascontiguousarray(x, dtype=np.float32).view(np.int32).astype(np.int64)
        return np.where(v < 0, -(v & 0x7FFFFFFF), v)
    return np.abs(ordinal(a) - ordinal(b))


@dataclass
class RouteCompare:
    heads: int = 0
    exact: int = 0
    near_cutoff: int = 0
    mismatched: List[str] = field(default_factory=list)

    def ok(self) -> bool:
        return not self.mismatched


def compare_route(r: zo.Route, gpu_levels: Dict[int, np.ndarray], gpu_leaves: np.ndarray,
                  out: RouteCompare, tag: str):
    """Per-level kept sets must be identical, except at and below a level whose oracle
    cutoff margin is below NEAR_CUTOFF (counted, not failed)."""
    out.heads += 1
    for lvl in range(r.top, 0, -1):
        sel = r.sel[lvl]
        want = sel.ids
        got = gpu_leaves if lvl == 1 else gpu_levels.get(lvl, np.zeros(0, np.int64))
        if len(want) == len(got) and np.array_equal(np.sort(got), want) and np.all(np.diff(got) > 0):
            continue
        if sel.margin < NEAR_CUTOFF:
            out.near_cutoff += 1
            return
        out.mismatched.append(f"{tag} level {lvl}: oracle m={sel.m} of {sel.n} (margin {sel.margin:.3g}), "
                              f"gpu kept {len(got)}; sym diff {len(np.setxor1d(want, got))}")
        return
    out.exact += 1
