"""GPU parity of the selector variants against the oracle's route with the same parameters:
zha_route_schedule (one top-p threshold per level, arXiv 2610.42112 §VII "Asymptotic length
scaling") and zha_route_topk (a fixed count per level, the budget K of App. D, Table VI).

The kept node sets of every level and the leaf lists must be identical, except at and below
a level whose oracle cutoff margin (top-p) or boundary gap (top-K) is under the near-cutoff
threshold (counted).  A constant schedule must give exactly the lists of zha_route with that p.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import zha_synth as S
from oracle import zha_oracle as zo
from tests.zha_cases import RouteCompare, compare_route, geometry, route_storage


pytestmark = pytest.mark.gpu

Z = None
DEV = "cuda"


def setup_module(module):
    global Z
    import hierarchical_sparse_attention_02_b200 as z
    z.load_library()
    Z = z


def _schedule(kind, p, depth):
    if kind == "root":
        return zo.p_root_schedule(p, depth)
    if kind == "leaf_only":
        return [p] + [1.0] * (depth - 1)
    if kind == "mixed":
        return [0.8 + 0.17 * i / max(1, depth - 1) for i in range(depth)]
    return [p] * depth


def _setup(w):
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    k_new, v_new = S.new_tokens(w, C, 1, DEV)
    q = S.queries(w, C, 1, DEV)
    tree = Z.empty_tree(g)
    tree.zero_()
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    Z.zha_append(g, K, V, k_new, v_new, w.T, qref, tree, st)   # the decode token at position T
    torch.cuda.synchronize()
    assert st.item() == 0
    return g, K, qref, q, tree, st


def _route(g, w, q, tree, st, ps, ks=None):
    nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
    level_cnt = torch.zeros(w.B, 1, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
    level_ids = torch.full((w.B, 1, w.Hq, max(nst, 1)), -1, dtype=torch.int32, device=DEV)
    ids = torch.full((w.B, 1, w.Hq, Z.leaf_cap(g)), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(w.B, 1, w.Hq, dtype=torch.int32, device=DEV)
    pos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE)
    if ks is not None:
        Z.zha_route_topk(g, q, pos, ks, tree, ids, cnt, ws, st, level_cnt, level_ids)
    elif isinstance(ps, float):
        Z.zha_route(g, q, pos, ps, tree, ids, cnt, ws, st, level_cnt, level_ids)
    else:
        Z.zha_route_schedule(g, q, pos, ps, tree, ids, cnt, ws, st, level_cnt, level_ids)
    torch.cuda.synchronize()
    assert st.item() == 0
    return ids.cpu().numpy(), cnt.cpu().numpy(), level_cnt.cpu().numpy(), level_ids.cpu().numpy()


@pytest.mark.parametrize("name,T,B,kind", [
    ("batched-decode-128k", 20000 + 7, 2, "root"),        # depth 3, p^(1/3) at every level
    ("batched-decode-128k", 20000 + 7, 2, "leaf_only"),   # p = 1 above the leaves
    ("batched-decode-128k", 70000 + 3, 1, "mixed"),       # distinct thresholds per level
    ("tiny-decode-f32", 8192, None, "mixed"),             # fp32 cache, depth 2
])
def test_route_schedule_parity(name, T, B, kind):
    base = S.workload(name)
    w = S.scaled(base, T=T, B=B, n_centres=min(base.n_centres, 1024))
    ps = _schedule(kind, w.p[0], w.depth)
    g, K, qref, q, tree, st = _setup(w)
    ids, cnt, lc, lids = _route(g, w, q, tree, st, ps)
    Kc = K.cpu()
    qr = qref.double().cpu().numpy()
    qc = q.double().cpu().numpy()
    cmp = RouteCompare()
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)][:4]
    for (b, hk) in units:
        otree = zo.build_tree(Kc[b, hk], w.T + 1, qr[hk], w.depth, route_storage=route_storage(w))
        for h in range(hk * w.G, (hk + 1) * w.G):
            levels, off = {}, 0
            for l in range(2, w.depth + 1):
                n = int(lc[b, 0, h, l - 1, 1])
                levels[l] = lids[b, 0, h, off:off + n].astype(np.int64)
                off += Z.tree_level(g, l).n_cap
            leaves = ids[b, 0, h, :int(cnt[b, 0, h])].astype(np.int64)
            compare_route(qc[b, 0, h], w.T, otree, ps, levels, leaves, cmp, f"b{b} h{h}")
    assert cmp.ok(), cmp.problems()
    assert cmp.exact > 0
    print(f"{w.name} {kind} {['%.4f' % x for x in ps]}: {cmp.summary()}")


def test_constant_schedule_is_zha_route():
    base = S.workload("batched-decode-128k")
    w = S.scaled(base, T=30000 + 1, B=2, n_centres=1024)
    g, K, qref, q, tree, st = _setup(w)
    p = w.p[0]
    a = _route(g, w, q, tree, st, p)
    b = _route(g, w, q, tree, st, [p] * w.depth)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def _workload(spec, T, B):
    base, _, ll = spec.partition("@L")
    w = S.scaled(S.workload(base), T=T, B=B, n_centres=min(S.workload(base).n_centres, 1024))
    return dataclasses.replace(w, depth=int(ll)) if ll else w


@pytest.mark.parametrize("spec,T,B,ks", [
    ("batched-decode-128k", 20000 + 7, 2, [64, 16, 4]),       # depth 3, a budget per level
    ("batched-decode-128k", 20000 + 7, 1, [100, 100, 100]),   # budgets above n at the upper levels
    ("tiny-decode-f32", 8192, None, [20, 3]),                  # fp32 cache, depth 2
    ("deep-tree-16m@L1", 1200000 + 5, None, [5000]),           # ~18.7K candidates: a cluster select
    ("deep-tree-16m@L1", 8700000 + 5, None, [20000]),          # ~136K candidates: the grid-wide chain
])
def test_route_topk_parity(spec, T, B, ks):
    w = _workload(spec, T, B)
    g, K, qref, q, tree, st = _setup(w)
    ids, cnt, lc, lids = _route(g, w, q, tree, st, None, ks)
    Kc = K.cpu()
    qr = qref.double().cpu().numpy()
    qc = q.double().cpu().numpy()
    cmp = RouteCompare()
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)][:3]
    for (b, hk) in units:
        otree = zo.build_tree(Kc[b, hk], w.T + 1, qr[hk], w.depth, route_storage=route_storage(w))
        for h in range(hk * w.G, (hk + 1) * w.G):
            levels = {}
            for l in range(2, w.depth + 1):
                o = sum(Z.tree_level(g, j).n_cap for j in range(2, l))
                levels[l] = lids[b, 0, h, o:o + int(lc[b, 0, h, l - 1, 1])].astype(np.int64)
            leaves = ids[b, 0, h, :int(cnt[b, 0, h])].astype(np.int64)
            compare_route(qc[b, 0, h], w.T, otree, 0.5, levels, leaves, cmp, f"b{b} h{h}", k=ks)
    assert cmp.ok(), cmp.problems()
    assert cmp.exact > 0
    print(f"{w.name} top-K {ks}: {cmp.summary()}")
