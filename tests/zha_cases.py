"""Shared harness of the GPU parity tests: seeded inputs on the device, the library
through its C ABI, and the CPU oracle on the same bytes (copied to the host)."""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

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


MAX_EXCUSED = 1 / 32    # fraction of the compared heads that may differ at a near cutoff (at least 1)

# every RouteCompare of the session with the test that made it; the terminal summary
# (tests/conftest.py) prints the GPU tests' tallies, so they show under `pytest -q`
ROUTE_REPORTS: List[Tuple[str, "RouteCompare"]] = []


@dataclass
class RouteCompare:
    """Per-test tally of the GPU's routes against the oracle's.

    exact       heads whose kept set equals the oracle's at every level
    near_cutoff heads that differ at some level where the oracle's cutoff is near (see
                ``near_cutoff_valid``); their levels below are compared with the oracle
                routed from the GPU's set, and their output with the oracle's attention
                over the GPU's leaf list
    near_levels (head, level) pairs whose oracle cutoff margin or boundary gap is under
                NEAR_CUTOFF, matched or not (how often the exemption could apply)
    mismatched  everything else: a failure
    """
    heads: int = 0
    exact: int = 0
    near_cutoff: int = 0
    near_levels: int = 0
    levels: int = 0
    mismatched: List[str] = field(default_factory=list)

    def __post_init__(self):
        test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" (")[0]
        ROUTE_REPORTS.append((test, self))

    def excused_limit(self) -> int:
        return max(1, int(self.heads * MAX_EXCUSED))

    def ok(self) -> bool:
        return not self.mismatched and self.near_cutoff <= self.excused_limit()

    def problems(self) -> List[str]:
        out = list(self.mismatched[:5])
        if self.near_cutoff > self.excused_limit():
            out.append(f"{self.near_cutoff} of {self.heads} heads differ at a near cutoff "
                       f"(limit {self.excused_limit()})")
        return out

    def summary(self) -> str:
        return (f"{self.exact} exact, {self.near_cutoff} near-cutoff mismatches of {self.heads} heads "
                f"({self.near_levels} of {self.levels} levels near the cutoff)")


def near_cutoff_valid(scores: np.ndarray, cand: np.ndarray, got: np.ndarray, p, k=None) -> str:
    """Whether ``got`` is a correct selection of the candidates ``cand`` (oracle scores
    ``scores``) up to the rounding the cutoff tolerance allows; '' if so, else why not.

    Top-p (threshold p): the set's softmax mass reaches p - NEAR_CUTOFF, dropping its
    smallest member leaves less than p + NEAR_CUTOFF, and no candidate left out has more
    softmax mass than a kept one by NEAR_CUTOFF or more (the boundary gap of the near-cutoff
    reading).  Top-K: |got| = min(K, n) and the same order condition.  p >= 1 keeps
    everything: no tolerance."""
    if len(np.unique(got)) != len(got) or not np.all(np.isin(got, cand)):
        return "kept ids are not distinct candidates"
    inside = np.isin(cand, got)
    if k is None and p >= 1.0:
        return "" if inside.all() else "p = 1 must keep every candidate"
    if not inside.any():
        return "" if len(cand) == 0 else "nothing kept"
    pi = np.exp(scores - scores.max())
    pi /= pi.sum()
    if k is None:
        mass = float(pi[inside].sum())
        if mass < p - NEAR_CUTOFF:
            return f"kept mass {mass:.6g} < p - {NEAR_CUTOFF}"
        if mass - float(pi[inside].min()) >= p + NEAR_CUTOFF:
            return f"not minimal: mass without the smallest kept {mass - pi[inside].min():.6g}"
    elif inside.sum() != min(int(k), len(cand)):
        return f"kept {int(inside.sum())} of {len(cand)}, K = {k}"
    if (~inside).any() and pi[~inside].max() - pi[inside].min() >= NEAR_CUTOFF:
        return (f"a dropped candidate has {pi[~inside].max() - pi[inside].min():.3g} more mass than a kept one "
                f"(scores {scores[~inside].max():.6g} > {scores[inside].min():.6g})")
    return ""


def compare_route(q: np.ndarray, t: int, tree: zo.Tree, p, gpu_levels: Dict[int, np.ndarray],
                  gpu_leaves: np.ndarray, out: RouteCompare, tag: str, k=None) -> np.ndarray:
    """Compare the GPU's kept sets of one query head, level by level from the top, with
    the oracle's.  Where they differ, the GPU's set must be a correct selection within
    the cutoff tolerance (``near_cutoff_valid``); the oracle then continues from the
    GPU's set (``zo.route(impose=...)``) and the levels below are compared with that.
    Returns the leaf list the head's output is to be checked against: the GPU's, which
    equals the oracle's unless the head is counted as a near-cutoff mismatch."""
    out.heads += 1
    scale = 1.0 / math.sqrt(q.shape[0])
    impose: Dict[int, np.ndarray] = {}
    r = zo.route(q, t, tree, p, k=k, impose=impose)
    for sel in r.sel.values():
        out.levels += 1
        out.near_levels += int(min(sel.margin, sel.gap) < NEAR_CUTOFF)
    differed = False
    for lvl in range(r.top, 0, -1):
        got = np.asarray(gpu_leaves if lvl == 1 else gpu_levels.get(lvl, np.zeros(0, np.int64)), np.int64)
        if len(got) > 1 and not np.all(np.diff(got) > 0):
            out.mismatched.append(f"{tag} level {lvl}: GPU ids not ascending")
            return got if lvl == 1 else r.leaves
        want = r.sel[lvl].ids
        if len(want) == len(got) and np.array_equal(got, want):
            continue
        scores = zo.node_scores(q, tree.levels[lvl - 1], r.cand[lvl], scale)
        why = near_cutoff_valid(scores, r.cand[lvl], got, zo._at_level(p, lvl) if k is None else None,
                                None if k is None else zo._at_level(k, lvl))
        if why:
            sel = r.sel[lvl]
            out.mismatched.append(f"{tag} level {lvl}: oracle m={sel.m} of {sel.n} (margin {sel.margin:.3g}), "
                                  f"gpu kept {len(got)}, sym diff {len(np.setxor1d(want, got))}: {why}")
            return gpu_leaves
        differed = True
        impose[lvl] = got
        r = zo.route(q, t, tree, p, k=k, impose=impose)   # the levels below, from the GPU's set
    if differed:
        out.near_cutoff += 1
    else:
        out.exact += 1
    return np.asarray(gpu_leaves, np.int64)
