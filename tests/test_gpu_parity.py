"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the same bytes.

Bars (per kernel):
  * tree summaries: bf16 k_hat within 1 bf16 ulp, fp32 k_hat within 1 fp32 ulp,
    b_hat within 1e-4 absolute, merge state within 1e-4 relative;
  * kept node sets at every level and the leaf lists: identical, except at and below a
    level whose oracle cutoff margin min(cum_m - p, p - cum_{m-1}) is under 1e-4
    (counted and reported);
  * outputs: bf16 max-abs <= 2e-2 and mean-abs <= 2e-3, fp32 max-abs <= 1e-4.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import zha_synth as S
from oracle import zha_oracle as zo
from tests.zha_cases import (RouteCompare, bf16_ulp_diff, compare_route, f32_ulp_diff, geometry,
                             route_storage, tree_arrays)

pytestmark = pytest.mark.gpu

Z = None


def setup_module(module):
    global Z
    import hierarchical_sparse_attention_02_b200 as z
    z.load_library()
    Z = z


DEV = "cuda"


def out_tol(w):
    return (1e-4, 1e-4) if w.dtype == "f32" else (2e-2, 2e-3)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------


class DecodeRun:
    """One decode step on the GPU plus everything the oracle needs."""

    def __init__(self, w: S.Workload, p: float, with_levels=True, k_transform=None):
        self.w, self.p = w, p
        self.g = g = geometry(w)
        self.C, self.K, self.V = S.clustered_kv(w, DEV)
        if k_transform is not None:
            k_transform(self.K)
        self.qref = S.reference_queries(w, DEV)
        self.k_new, self.v_new = S.new_tokens(w, self.C, 1, DEV)
        self.q = S.queries(w, self.C, 1, DEV)
        self.tree = Z.empty_tree(g)
        self.tree.zero_()
        self.ws = Z.empty_workspace(g, 1, Z.ZHA_OP_DECODE)
        self.st = torch.zeros(1, dtype=torch.int32, device=DEV)
        Z.zha_build_tree(g, self.K, w.T, self.qref, self.tree, self.st)
        cap = Z.leaf_cap(g)
        self.leaf_ids = torch.full((w.B, 1, w.Hq, cap), -7, dtype=torch.int32, device=DEV)
        self.leaf_cnt = torch.zeros(w.B, 1, w.Hq, dtype=torch.int32, device=DEV)
        self.O = torch.empty(w.B, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
        Z.zha_decode(g, self.q, self.k_new, self.v_new, self.K, self.V, w.T, self.qref, p, self.tree,
                     self.leaf_ids, self.leaf_cnt, self.O, self.ws, self.st)
        torch.cuda.synchronize()
        assert self.st.item() == 0, Z.ZhaError("device", self.st.item())
        self.levels = None
        if with_levels:
            self.route_levels()

    def route_levels(self):
        g, w = self.g, self.w
        nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
        self.level_cnt = torch.zeros(w.B, 1, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
        self.level_ids = torch.full((w.B, 1, w.Hq, max(nst, 1)), -1, dtype=torch.int32, device=DEV)
        lid = torch.full_like(self.leaf_ids, -7)
        lcnt = torch.zeros_like(self.leaf_cnt)
        pos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=DEV)
        ws = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE)
        Z.zha_route(g, self.q, pos, self.p, self.tree, lid, lcnt, ws, self.st, self.level_cnt, self.level_ids)
        torch.cuda.synchronize()
        assert self.st.item() == 0
        # the stand-alone route must agree with the one inside zha_decode
        assert torch.equal(lcnt, self.leaf_cnt)
        for b in range(w.B):
            for h in range(w.Hq):
                n = int(lcnt[b, 0, h])
                assert torch.equal(lid[b, 0, h, :n], self.leaf_ids[b, 0, h, :n])
        self.levels = True

    def gpu_levels(self, b, h):
        out = {}
        off = 0
        for l in range(2, self.w.depth + 1):
            n = int(self.level_cnt[b, 0, h, l - 1, 1])
            out[l] = self.level_ids[b, 0, h, off:off + n].cpu().numpy().astype(np.int64)
            off += Z.tree_level(self.g, l).n_cap
        return out

    def gpu_leaves(self, b, h):
        n = int(self.leaf_cnt[b, 0, h])
        return self.leaf_ids[b, 0, h, :n].cpu().numpy().astype(np.int64)


def check_decode(run: DecodeRun, units, heads_per_unit=None):
    """Oracle on the chosen (b, h_kv) units; returns the routing comparison.  Every head's
    output is checked against the oracle's attention over the head's GPU leaf list (the
    oracle's own list unless the head differs at a near cutoff, see compare_route)."""
    w = run.w
    Kc, Vc = run.K.cpu(), run.V.cpu()
    qref = run.qref.double().cpu().numpy()
    q = run.q.double().cpu().numpy()
    O = run.O.float().cpu().numpy()
    cmp = RouteCompare()
    errs = []
    for (b, hk) in units:
        tree = zo.build_tree(Kc[b, hk], w.T + 1, qref[hk], w.depth, route_storage=route_storage(w))
        heads = range(hk * w.G, (hk + 1) * w.G) if heads_per_unit is None else \
            [hk * w.G + i for i in heads_per_unit]
        for h in heads:
            leaves = compare_route(q[b, 0, h], w.T, tree, run.p, run.gpu_levels(b, h), run.gpu_leaves(b, h),
                                   cmp, f"b{b} h{h}")
            o, _ = zo.attention(q[b, 0, h], Kc[b, hk], Vc[b, hk], zo.index_set(leaves, w.T))
            errs.append(np.abs(O[b, 0, h] - o))
    assert cmp.ok(), cmp.problems()
    assert errs, "no head compared"
    e = np.stack(errs)
    mx, mean = out_tol(w)
    assert e.max() <= mx and e.mean() <= mean, (e.max(), e.mean())
    return cmp


# ---------------------------------------------------------------------------
# tree build
# ---------------------------------------------------------------------------


def _check_tree(w, K, qref, tree, T, units):
    g = geometry(w)
    Kc = K.cpu()
    for (b, hk) in units:
        ot = zo.build_tree(Kc[b, hk], T, qref[hk].double().cpu().numpy(), w.depth, route_storage=route_storage(w))
        for lvl in range(1, w.depth + 1):
            kr, bh, F, ks = tree_arrays(g, tree, lvl)
            L = ot.levels[lvl - 1]
            n = L.n
            if n == 0:
                continue
            gk = kr[b, hk, :n].float().cpu().numpy()
            if w.dtype == "bf16":
                ulp = bf16_ulp_diff(gk, L.k_route)
            else:
                ulp = f32_ulp_diff(gk, L.k_route)
            assert ulp.max() <= 1, (lvl, ulp.max())
            assert np.abs(bh[b, hk, :n].cpu().numpy() - L.b_hat).max() <= 1e-4
            assert f32_ulp_diff(ks[b, hk, :n].cpu().numpy(), L.k_state).max() <= 1
            np.testing.assert_allclose(F[b, hk, :n].cpu().numpy(), L.F, rtol=1e-4, atol=0)


@pytest.mark.parametrize("name,T,B,R", [("tiny-decode-f32", 8192, None, 4), ("batched-decode-128k", 16384 + 64 * 5, 2, 4),
                                        ("deep-tree-16m", 70000, None, 4), ("batched-decode-128k", 20000, 1, 1),
                                        ("batched-decode-128k", 20000, 1, 16), ("tiny-decode-f32", 8192, None, 16)])
def test_tree_build_parity(name, T, B, R):
    import dataclasses
    w = S.scaled(S.workload(name), T=T, B=B, n_centres=min(S.workload(name).n_centres, 1024))
    w = dataclasses.replace(w, R=R)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    tree = Z.empty_tree(g)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_build_tree(g, K, T, qref, tree, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    _check_tree(w, K, qref, tree, T, [(b, h) for b in range(w.B) for h in range(w.Hkv)])


def test_append_equals_rebuild():
    w = S.scaled(S.workload("prefill-append-256k"), T=16384 - 100, n_new=1300, n_centres=512)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    t1 = Z.empty_tree(g); t1.zero_()
    Z.zha_build_tree(g, K, w.T, qref, t1, st)
    # append in uneven pieces crossing leaf and level-2 boundaries
    t = w.T
    for piece in (1, 63, 500, 736):
        kn, vn = S.new_tokens(w, C, piece, DEV, step=t)
        Z.zha_append(g, K, V, kn, vn, t, qref, t1, st)
        t += piece
    t2 = Z.empty_tree(g); t2.zero_()
    Z.zha_build_tree(g, K, t, qref, t2, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(t1, t2)
    _check_tree(w, K, qref, t1, t, [(0, 0), (0, 1)])


# ---------------------------------------------------------------------------
# decode: append + route + sparse attention
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("name,T,B,p", [
    ("tiny-decode-f32", 8192, None, 0.9),
    ("tiny-decode-f32", 8192, None, 0.5),
    ("batched-decode-128k", 32768, 2, 0.95),
    ("long-decode-1m", 65536 + 64 * 7 + 63, 1, 0.99),    # the new token completes a leaf
    ("long-decode-1m", 65536 + 37, 1, 0.95),             # a partial chunk of 38 keys
    ("deep-tree-16m", 300000, None, 0.95),               # empty top levels
    ("batched-decode-128k@R1", 32768, 1, 0.95),
    ("batched-decode-128k@R16", 32768, 1, 0.9),
    ("deep-tree-16m@L1", 1200000 + 5, None, 0.95),       # one level: ~18.7K candidates per head
    ("deep-tree-16m@L2", 1200000, None, 0.99),           # > 16K leaf candidates below the top
    ("deep-tree-16m@L1", 2300000 + 5, None, 0.95),       # ~36K candidates: a 4-CTA cluster select
    ("deep-tree-16m@L1", 4500000 + 5, None, 0.95),       # ~70K candidates: an 8-CTA cluster select
    ("batched-decode-128k", 180000 + 9, 8, 0.95),        # 2813 candidates x 256 heads: 256-thread CTAs
])
def test_decode_parity(name, T, B, p):
    import dataclasses
    base, _, rr = name.partition("@R")
    base, _, ll = base.partition("@L")
    w = S.scaled(S.workload(base), T=T, B=B, n_centres=min(S.workload(base).n_centres, 1024))
    if rr:
        w = dataclasses.replace(w, R=int(rr))
    if ll:
        w = dataclasses.replace(w, depth=int(ll))
    run = DecodeRun(w, p)
    units = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    cmp = check_decode(run, units if len(units) <= 8 else [units[0], units[len(units) // 2], units[-1]])
    print(f"{w.name} p={p}: {cmp.summary()}")


def test_decode_p1_is_dense():
    w = S.scaled(S.workload("batched-decode-128k"), T=8192 + 11, B=1, n_centres=256)
    run = DecodeRun(w, 1.0)
    n1 = (w.T // 64)
    assert (run.leaf_cnt == n1).all()
    g = run.g
    pos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=DEV)
    O2 = torch.empty_like(run.O)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_DENSE)
    Z.zha_dense_decode(g, run.q, run.K, run.V, pos, O2, ws, run.st)
    torch.cuda.synchronize()
    assert (O2.float() - run.O.float()).abs().max().item() <= 2e-2
    check_decode(run, [(0, h) for h in range(w.Hkv)])


@pytest.mark.parametrize("name,T,p", [("batched-decode-128k", 16384 + 64 * 3 + 17, 0.9),
                                      ("batched-decode-128k", 70000 + 17, 0.95),
                                      ("deep-tree-16m@L1", 1200000 + 5, 0.9)])
def test_decode_tied_chunks(name, T, p):
    """Leaf chunks repeated with period 5: exact score ties at level 1 (and, with period 5
    over the parents, at level 2), boundaries inside tie groups; the select must keep the
    lowest ids of a tie group like the oracle.  The three cases put level 1 on the warp
    select (259 candidates), a 1024-thread CTA (1094) and a 2-CTA cluster (18750
    candidates in 5 tie groups of 3750: the tie ranks run across the cluster)."""
    import dataclasses
    base, _, ll = name.partition("@L")
    w = S.scaled(S.workload(base), T=T, B=1, n_centres=256)
    if ll:
        w = dataclasses.replace(w, depth=int(ll))

    def tie(K):
        n = w.T // 64
        src = torch.arange(n, device=K.device) % 5
        Kv = K[:, :, :n * 64].view(K.shape[0], K.shape[1], n, 64, K.shape[-1])
        Kv.copy_(Kv[:, :, src].clone())

    run = DecodeRun(w, p, k_transform=tie)
    cmp = check_decode(run, [(0, h) for h in range(w.Hkv)])
    print(f"tied chunks T={T} p={p}: {cmp.summary()}")


def test_decode_is_deterministic():
    w = S.scaled(S.workload("batched-decode-128k"), T=16384, B=2, n_centres=512)
    a = DecodeRun(w, 0.95, with_levels=False)
    b = DecodeRun(w, 0.95, with_levels=False)
    assert torch.equal(a.leaf_cnt, b.leaf_cnt)
    assert torch.equal(a.O, b.O)
    assert torch.equal(a.tree, b.tree)


# ---------------------------------------------------------------------------
# sparse attention fed by the oracle's own leaf lists
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("name,T", [("tiny-decode-f32", 8192 + 5), ("batched-decode-128k", 20000)])
def test_sparse_attn_on_oracle_lists(name, T):
    w = S.scaled(S.workload(name), T=T, B=1, n_centres=256)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    q = S.queries(w, C, 3, DEV)                                     # 3 queries per sequence
    pos_np = np.array([[T - 1, T - 64, 70]])
    rng = np.random.default_rng(0)
    cap = Z.leaf_cap(g)
    ids = np.full((1, 3, w.Hq, cap), -1, np.int32)
    cnt = np.zeros((1, 3, w.Hq), np.int32)
    for qi in range(3):
        nvis = (pos_np[0, qi] // 64)
        for h in range(w.Hq):
            k = int(rng.integers(0, nvis + 1))
            sel = np.sort(rng.choice(nvis, size=k, replace=False)) if k else np.zeros(0, int)
            ids[0, qi, h, :k] = sel
            cnt[0, qi, h] = k
    O = torch.empty(1, 3, w.Hq, w.d, dtype=g.dtype, device=DEV)
    lse = torch.empty(1, 3, w.Hq, dtype=torch.float32, device=DEV)
    ws = Z.empty_workspace(g, 3, Z.ZHA_OP_ATTN)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_sparse_attn(g, q, K, V, torch.from_numpy(pos_np).to(DEV), torch.from_numpy(ids).to(DEV),
                      torch.from_numpy(cnt).to(DEV), O, ws, st, lse=lse)
    torch.cuda.synchronize()
    assert st.item() == 0
    Kc, Vc, qc = K.cpu(), V.cpu(), q.double().cpu().numpy()
    mx, mean = out_tol(w)
    errs = []
    for qi in range(3):
        for h in range(w.Hq):
            idx = zo.index_set(ids[0, qi, h, :cnt[0, qi, h]], int(pos_np[0, qi]))
            o, l = zo.attention(qc[0, qi, h], Kc[0, h // w.G], Vc[0, h // w.G], idx)
            errs.append(np.abs(O[0, qi, h].float().cpu().numpy() - o))
            assert abs(lse[0, qi, h].item() - l) <= 1e-3 * max(1.0, abs(l))
    e = np.stack(errs)
    assert e.max() <= mx and e.mean() <= mean, (e.max(), e.mean())


# ---------------------------------------------------------------------------
# baselines
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("name,T", [("tiny-decode-f32", 8192), ("batched-decode-128k", 20000 + 17),
                                    ("batched-decode-128k", 140000 + 3)])   # > 128 splits: CTA combine
def test_dense_decode_parity(name, T):
    w = S.scaled(S.workload(name), T=T, B=2, n_centres=256)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    q = S.queries(w, C, 2, DEV)
    pos_np = np.array([[T - 1, 100]] * w.B)
    O = torch.empty(w.B, 2, w.Hq, w.d, dtype=g.dtype, device=DEV)
    ws = Z.empty_workspace(g, 2, Z.ZHA_OP_DENSE)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_dense_decode(g, q, K, V, torch.from_numpy(pos_np).to(DEV), O, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Kc, Vc, qc = K.cpu(), V.cpu(), q.double().cpu().numpy()
    errs = []
    for b in range(w.B):
        for qi in range(2):
            for h in range(w.Hq):
                o, _ = zo.dense_attention(qc[b, qi, h], Kc[b, h // w.G], Vc[b, h // w.G], int(pos_np[b, qi]))
                errs.append(np.abs(O[b, qi, h].float().cpu().numpy() - o))
    e = np.stack(errs)
    mx, mean = out_tol(w)
    assert e.max() <= mx and e.mean() <= mean, (e.max(), e.mean())


def test_flat_index_parity():
    w = S.scaled(S.workload("long-decode-1m"), T=32768 + 64, B=1, n_centres=512)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    q = S.queries(w, C, 1, DEV)
    pos = torch.full((1, 1), w.T - 1, dtype=torch.int64, device=DEV)
    cap = Z.leaf_cap(g)
    ids = torch.full((1, 1, w.Hq, cap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, 1, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(1, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_FLAT)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_flat_index(g, q, K, V, pos, 0.95, ids, cnt, O, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Kc, Vc, qc = K.cpu(), V.cpu(), q.double().cpu().numpy()
    t = w.T - 1
    exact = 0
    for h in range(w.Hq):
        sel = zo.flat_select(qc[0, 0, h], Kc[0, h // w.G], t, 0.95)
        got = ids[0, 0, h, :int(cnt[0, 0, h])].cpu().numpy()
        # fp32 chunk log-masses: sets may differ only among near-equal scores at the boundary
        diff = np.setxor1d(sel.ids, got)
        if len(diff) == 0:
            exact += 1
            o, _ = zo.attention(qc[0, 0, h], Kc[0, h // w.G], Vc[0, h // w.G], zo.index_set(sel.ids, t))
            assert np.abs(O[0, 0, h].float().cpu().numpy() - o).max() <= 2e-2
        else:
            s = zo.flat_scores(qc[0, 0, h], Kc[0, h // w.G], t)
            order = np.sort(s)[::-1]
            boundary = order[sel.m - 1]
            assert np.abs(s[diff] - boundary).max() <= 1e-4 or sel.margin < 1e-4, (h, len(diff))
    assert exact >= w.Hq // 2


# ---------------------------------------------------------------------------
# chunked prefill with incremental append (causal routing)
# ---------------------------------------------------------------------------


def test_prefill_append_causal_parity():
    w = S.scaled(S.workload("prefill-append-256k"), T=20000, n_new=512, n_centres=512)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tree = Z.empty_tree(g)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    kn, vn = S.new_tokens(w, C, w.n_new, DEV)
    Z.zha_append(g, K, V, kn, vn, w.T, qref, tree, st)
    Q = S.queries(w, C, w.n_new, DEV)
    pos = (w.T + torch.arange(w.n_new, device=DEV, dtype=torch.int64)).view(1, -1)
    cap = Z.leaf_cap(g)
    ids = torch.full((1, w.n_new, w.Hq, cap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, w.n_new, w.Hq, dtype=torch.int32, device=DEV)
    nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
    lcnt = torch.zeros(1, w.n_new, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
    lids = torch.full((1, w.n_new, w.Hq, nst), -1, dtype=torch.int32, device=DEV)
    ws = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_ROUTE)
    Z.zha_route(g, Q, pos, 0.95, tree, ids, cnt, ws, st, lcnt, lids)
    O = torch.empty(1, w.n_new, w.Hq, w.d, dtype=g.dtype, device=DEV)
    wa = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_ATTN)
    Z.zha_sparse_attn(g, Q, K, V, pos, ids, cnt, O, wa, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    Kc, Vc = K.cpu(), V.cpu()
    qc = Q.double().cpu().numpy()
    qr = qref.double().cpu().numpy()
    trees = {hk: zo.build_tree(Kc[0, hk], w.T + w.n_new, qr[hk], w.depth) for hk in range(w.Hkv)}
    cmp = RouteCompare()
    errs = []
    rng = np.random.default_rng(1)
    for qi in sorted(set(rng.integers(0, w.n_new, 24).tolist()) | {0, w.n_new - 1}):
        t = w.T + qi
        for h in range(w.Hq):
            hk = h // w.G
            off, lv = 0, {}
            for l in range(2, w.depth + 1):
                n = int(lcnt[0, qi, h, l - 1, 1])
                lv[l] = lids[0, qi, h, off:off + n].cpu().numpy().astype(np.int64)
                off += Z.tree_level(g, l).n_cap
            got = ids[0, qi, h, :int(cnt[0, qi, h])].cpu().numpy().astype(np.int64)
            leaves = compare_route(qc[0, qi, h], t, trees[hk], 0.95, lv, got, cmp, f"q{qi} h{h}")
            o, _ = zo.attention(qc[0, qi, h], Kc[0, hk], Vc[0, hk], zo.index_set(leaves, t))
            errs.append(np.abs(O[0, qi, h].float().cpu().numpy() - o))
    assert cmp.ok(), cmp.problems()
    e = np.stack(errs)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3
    print(f"prefill: {cmp.summary()}")


# ---------------------------------------------------------------------------
# edge cases and device-side errors
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("T", [0, 10, 63, 64, 65, 1024 + 63])
def test_short_caches(T):
    w = S.scaled(S.workload("batched-decode-128k"), T=T, B=1, n_centres=64)
    run = DecodeRun(w, 0.95)
    nvis = T // 64
    assert (run.leaf_cnt <= nvis).all()
    if nvis == 0:
        assert (run.leaf_cnt == 0).all()
    check_decode(run, [(0, h) for h in range(w.Hkv)])


def test_leaf_cap_overflow_sets_status():
    w = S.scaled(S.workload("batched-decode-128k"), T=8192, B=1, n_centres=64)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    q = S.queries(w, C, 1, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tree = Z.empty_tree(g)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    ids = torch.full((1, 1, w.Hq, 4), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, 1, w.Hq, dtype=torch.int32, device=DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE)
    pos = torch.full((1, 1), w.T - 1, dtype=torch.int64, device=DEV)
    Z.zha_route(g, q, pos, 1.0, tree, ids, cnt, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 3                    # ZHA_ERR_CAPACITY
    assert (cnt == 4).all()
    assert (ids >= 0).all()


def test_bad_position_sets_status():
    w = S.scaled(S.workload("batched-decode-128k"), T=4096, B=1, n_centres=64)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    q = S.queries(w, C, 1, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tree = Z.empty_tree(g)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    ids = torch.full((1, 1, w.Hq, Z.leaf_cap(g)), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, 1, w.Hq, dtype=torch.int32, device=DEV)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE)
    pos = torch.full((1, 1), g.t_cap + 5, dtype=torch.int64, device=DEV)
    Z.zha_route(g, q, pos, 0.9, tree, ids, cnt, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 1                    # ZHA_ERR_INVALID_ARG
    assert (cnt == 0).all()
