"""Parity at the workloads' full sizes, in the launch configuration the benchmark times.

Each test runs the whole batch on the GPU exactly as bench.py does (zha_build_tree, then
zha_decode for one new token per sequence; chunked prefill: zha_append + zha_route +
zha_sparse_attn for 4096 causal queries), then checks sampled (sequence, KV head) units
or sampled queries against the CPU oracle one head at a time: every level's kept set
(identical except near-cutoff levels, counted), the leaf list and the output.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import zha_synth as S
from oracle import zha_oracle as zo
from tests.zha_cases import RouteCompare, compare_route, geometry, route_storage

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def Z():
    import hierarchical_sparse_attention_02_b200 as z
    z.load_library()
    return z


def _decode_full(Z, w, p):
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    k_new, v_new = S.new_tokens(w, C, 1, DEV)
    q = S.queries(w, C, 1, DEV)
    del C
    tree = Z.empty_tree(g, DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_DECODE, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    cap = Z.leaf_cap(g)
    ids = torch.empty(w.B, 1, w.Hq, cap, dtype=torch.int32, device=DEV)
    cnt = torch.empty(w.B, 1, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(w.B, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
    Z.zha_decode(g, q, k_new, v_new, K, V, w.T, qref, p, tree, ids, cnt, O, ws, st)
    # per-level kept sets of the same routing (bit-identical to the one inside zha_decode)
    nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
    lcnt = torch.zeros(w.B, 1, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
    lids = torch.full((w.B, 1, w.Hq, max(nst, 1)), -1, dtype=torch.int32, device=DEV)
    ids2 = torch.empty_like(ids)
    cnt2 = torch.empty_like(cnt)
    pos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=DEV)
    del ws
    wsr = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE, DEV)
    Z.zha_route(g, q, pos, p, tree, ids2, cnt2, wsr, st, lcnt, lids)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(cnt, cnt2)
    return g, K, V, q, qref, ids, cnt, O, lcnt, lids


def _check_units(Z, w, p, g, K, V, q, qref, ids, cnt, O, lcnt, lids, units, heads=None):
    cmp = RouteCompare()
    errs = []
    qc = q.double().cpu().numpy()
    qr = qref.double().cpu().numpy()
    for (b, hk) in units:
        Kc, Vc = K[b, hk].cpu(), V[b, hk].cpu()
        tree = zo.build_tree(Kc, w.T + 1, qr[hk], w.depth, route_storage=route_storage(w))
        hs = range(hk * w.G, (hk + 1) * w.G) if heads is None else [hk * w.G + i for i in heads]
        for h in hs:
            lv, off = {}, 0
            for l in range(2, w.depth + 1):
                n = int(lcnt[b, 0, h, l - 1, 1])
                lv[l] = lids[b, 0, h, off:off + n].cpu().numpy().astype(np.int64)
                off += Z.tree_level(g, l).n_cap
            got = ids[b, 0, h, :int(cnt[b, 0, h])].cpu().numpy().astype(np.int64)
            leaves = compare_route(qc[b, 0, h], w.T, tree, p, lv, got, cmp, f"b{b} h{h}")
            o, _ = zo.attention(qc[b, 0, h], Kc, Vc, zo.index_set(leaves, w.T))
            errs.append(np.abs(O[b, 0, h].float().cpu().numpy() - o))
    assert cmp.ok(), cmp.problems()
    e = np.stack(errs)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())
    print(f"{w.name} p={p}: {cmp.summary()}; max err {e.max():.2e}")


def test_batched_decode_128k_full(Z):
    w = S.workload("batched-decode-128k")
    out = _decode_full(Z, w, w.p[0])
    _check_units(Z, w, w.p[0], *out, units=[(0, 0), (31, 3)])


@pytest.mark.parametrize("p", [0.95, 0.99])
def test_long_decode_1m_full(Z, p):
    w = S.workload("long-decode-1m")
    out = _decode_full(Z, w, p)
    _check_units(Z, w, p, *out, units=[(0, 1), (3, 3)], heads=[0, 5])


def test_deep_tree_16m_full(Z):
    w = S.workload("deep-tree-16m")
    out = _decode_full(Z, w, w.p[0])
    _check_units(Z, w, w.p[0], *out, units=[(0, 0)], heads=[0, 7])


def test_prefill_append_256k_full(Z):
    w = S.workload("prefill-append-256k")
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tree = Z.empty_tree(g, DEV)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    kn, vn = S.new_tokens(w, C, w.n_new, DEV)
    Z.zha_append(g, K, V, kn, vn, w.T, qref, tree, st)
    Q = S.queries(w, C, w.n_new, DEV)
    pos = (w.T + torch.arange(w.n_new, device=DEV, dtype=torch.int64)).view(1, -1)
    cap = Z.leaf_cap(g)
    ids = torch.empty(1, w.n_new, w.Hq, cap, dtype=torch.int32, device=DEV)
    cnt = torch.empty(1, w.n_new, w.Hq, dtype=torch.int32, device=DEV)
    nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
    lcnt = torch.zeros(1, w.n_new, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
    lids = torch.full((1, w.n_new, w.Hq, nst), -1, dtype=torch.int32, device=DEV)
    ws = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_ROUTE, DEV)
    Z.zha_route(g, Q, pos, w.p[0], tree, ids, cnt, ws, st, lcnt, lids)
    del ws
    O = torch.empty(1, w.n_new, w.Hq, w.d, dtype=g.dtype, device=DEV)
    wa = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_ATTN, DEV)
    Z.zha_sparse_attn(g, Q, K, V, pos, ids, cnt, O, wa, st)
    del wa
    # the same attention per query tile on the tensor cores (the launch bench.py times)
    Ot = torch.empty_like(O)
    wp = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_PREFILL, DEV)
    Z.zha_prefill_attn(g, Q, K, V, pos, ids, cnt, Ot, wp, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    d = (Ot.float() - O.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3, (d.max().item(), d.mean().item())
    qc = Q.double().cpu().numpy()
    qr = qref.double().cpu().numpy()
    Kc = [K[0, hk].cpu() for hk in range(w.Hkv)]
    Vc = [V[0, hk].cpu() for hk in range(w.Hkv)]
    trees = [zo.build_tree(Kc[hk], w.T + w.n_new, qr[hk], w.depth) for hk in range(w.Hkv)]
    cmp = RouteCompare()
    errs = []
    rng = np.random.default_rng(7)
    for qi in sorted(set(rng.integers(0, w.n_new, 6).tolist()) | {0, 63, 64, w.n_new - 1}):
        t = w.T + qi
        for h in (0, 9, 15):
            hk = h // w.G
            lv, off = {}, 0
            for l in range(2, w.depth + 1):
                n = int(lcnt[0, qi, h, l - 1, 1])
                lv[l] = lids[0, qi, h, off:off + n].cpu().numpy().astype(np.int64)
                off += Z.tree_level(g, l).n_cap
            got = ids[0, qi, h, :int(cnt[0, qi, h])].cpu().numpy().astype(np.int64)
            leaves = compare_route(qc[0, qi, h], t, trees[hk], w.p[0], lv, got, cmp, f"q{qi} h{h}")
            o, _ = zo.attention(qc[0, qi, h], Kc[hk], Vc[hk], zo.index_set(leaves, t))
            errs.append(np.abs(O[0, qi, h].float().cpu().numpy() - o))
            errs.append(np.abs(Ot[0, qi, h].float().cpu().numpy() - o))
    assert cmp.ok(), cmp.problems()
    e = np.stack(errs)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())
    print(f"prefill-append-256k: {cmp.summary()}")


@pytest.mark.parametrize("name,units,heads", [("batched-decode-128k", [(0, 0), (31, 3)], None),
                                              ("long-decode-1m", [(2, 1)], [0, 5])])
def test_flat_index_full(Z, name, units, heads):
    """The flat exact-LSE indexer at full size: tensor-core chunk scores over every visible
    chunk, top-p select, sparse attention; sampled heads against the oracle's exact chunk
    scores (fp32 chunk log-masses: sets may differ only among near-equal scores at the
    boundary)."""
    w = S.workload(name)
    g = geometry(w)
    p = w.p[0]
    C, K, V = S.clustered_kv(w, DEV)
    q = S.queries(w, C, 1, DEV)
    del C
    t = w.T - 1
    pos = torch.full((w.B, 1), t, dtype=torch.int64, device=DEV)
    cap = Z.leaf_cap(g)
    ids = torch.full((w.B, 1, w.Hq, cap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(w.B, 1, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(w.B, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_FLAT, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_flat_index(g, q, K, V, pos, p, ids, cnt, O, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    qc = q.double().cpu().numpy()
    exact = total = 0
    for (b, hk) in units:
        Kc, Vc = K[b, hk].cpu(), V[b, hk].cpu()
        hs = range(hk * w.G, (hk + 1) * w.G) if heads is None else [hk * w.G + i for i in heads]
        for h in hs:
            total += 1
            sel = zo.flat_select(qc[b, 0, h], Kc, t, p)
            got = ids[b, 0, h, :int(cnt[b, 0, h])].cpu().numpy()
            diff = np.setxor1d(sel.ids, got)
            if len(diff) == 0:
                exact += 1
                o, _ = zo.attention(qc[b, 0, h], Kc, Vc, zo.index_set(sel.ids, t))
                assert np.abs(O[b, 0, h].float().cpu().numpy() - o).max() <= 2e-2
            else:
                s = zo.flat_scores(qc[b, 0, h], Kc, t)
                boundary = np.sort(s)[::-1][sel.m - 1]
                assert np.abs(s[diff] - boundary).max() <= 1e-4 or sel.margin < 1e-4, (b, h, len(diff))
    assert exact >= total // 2
    print(f"{name} flat: {exact} exact of {total} heads")


@pytest.mark.parametrize("tie", [False, True])
def test_flat_index_wide(Z, tie):
    """The flat indexer over 8.7 M keys of one KV head: ~136 K candidate chunks per query
    head, beyond what the clusters hold in shared memory, so the select runs as the chain
    of grid-wide kernels over (head, chunk).  With tied chunks (period 5) every score comes
    in groups of ~27 K equal values spread over all chunks and the boundary falls inside a
    group: the lowest ids of the group must be kept, exactly as the oracle keeps them."""
    w = S.scaled(S.workload("deep-tree-16m"), T=8_700_000 + 37, B=1)
    g = geometry(w)
    p = w.p[0]
    C, K, V = S.clustered_kv(w, DEV)
    q = S.queries(w, C, 1, DEV)
    del C
    if tie:
        n = w.T // 64
        src = torch.arange(n, device=DEV) % 5
        Kv = K[:, :, :n * 64].view(K.shape[0], K.shape[1], n, 64, K.shape[-1])
        Kv.copy_(Kv[:, :, src].clone())
    t = w.T - 1
    pos = torch.full((w.B, 1), t, dtype=torch.int64, device=DEV)
    cap = Z.leaf_cap(g)
    assert cap > 8 * 16896                             # beyond the cluster selects
    ids = torch.full((w.B, 1, w.Hq, cap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(w.B, 1, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(w.B, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_FLAT, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_flat_index(g, q, K, V, pos, p, ids, cnt, O, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    qc = q.double().cpu().numpy()
    Kc = K[0, 0].cpu()
    del V, ws
    exact = 0
    for h in (0, 5):
        sel = zo.flat_select(qc[0, 0, h], Kc, t, p)
        got = ids[0, 0, h, :int(cnt[0, 0, h])].cpu().numpy()
        diff = np.setxor1d(sel.ids, got)
        if tie:
            assert len(diff) == 0, (h, len(diff), len(sel.ids), len(got))
        elif len(diff):
            s = zo.flat_scores(qc[0, 0, h], Kc, t)
            boundary = np.sort(s)[::-1][sel.m - 1]
            assert np.abs(s[diff] - boundary).max() <= 1e-4 or sel.margin < 1e-4, (h, len(diff))
        exact += len(diff) == 0
    print(f"flat wide (tie={tie}): {exact} exact of 2 heads, {int(cnt[0, 0, 0])} chunks kept of {t // 64}")
