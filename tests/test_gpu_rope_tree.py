"""GPU parity of the rotary-position tree (arXiv 2610.42112 §III-B: references rotated to
each node's last position, children re-anchored before the merge) against the oracle's
build_tree(..., inv_freq=...), on the same keys, reference queries and frequency table.

Bars as for the plain tree: bf16 k_hat within 1 bf16 ulp (fp32: 1 fp32 ulp), b_hat within
1e-4, merge state within 1 fp32 ulp / 1e-4 relative; append equals rebuild bit for bit; a
decode step over the rotary tree keeps the oracle's node sets (near-cutoff levels counted)
and its outputs meet the attention bars.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import zha_synth as S
from oracle import zha_oracle as zo
from tests.zha_cases import (RouteCompare, bf16_ulp_diff, compare_route, f32_ulp_diff, route_storage,
                             tree_arrays)

pytestmark = pytest.mark.gpu

Z = None
DEV = "cuda"


def setup_module(module):
    global Z
    import hierarchical_sparse_attention_02_b200 as z
    z.load_library()
    Z = z


def rope_table(h: int, base: float = 10000.0) -> torch.Tensor:
    """The usual RoPE frequencies over 2h rotated dims, f_i = base^(-i/h), as fp32."""
    return (base ** (-torch.arange(h, dtype=torch.float64) / h)).float()


def rope_geometry(w: S.Workload, h: int):
    return Z.Geometry(B=w.B, Hq=w.Hq, Hkv=w.Hkv, t_cap=w.t_cap, depth=w.depth, R=w.R, d=w.d, leaf=w.leaf,
                      branch=w.branch, dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                      rope_pairs=h)


def check_tree(w, g, K, qref, freq, tree, T, units):
    Kc = K.cpu()
    f = freq.double().numpy()
    for (b, hk) in units:
        ot = zo.build_tree(Kc[b, hk], T, qref[hk].double().cpu().numpy(), w.depth,
                           route_storage=route_storage(w), inv_freq=f)
        for lvl in range(1, w.depth + 1):
            kr, bh, F, ks = tree_arrays(g, tree, lvl)
            L = ot.levels[lvl - 1]
            n = L.n
            if n == 0:
                continue
            gk = kr[b, hk, :n].float().cpu().numpy()
            ulp = bf16_ulp_diff(gk, L.k_route) if w.dtype == "bf16" else f32_ulp_diff(gk, L.k_route)
            assert ulp.max() <= 1, (lvl, ulp.max())
            assert np.abs(bh[b, hk, :n].cpu().numpy() - L.b_hat).max() <= 1e-4, lvl
            assert f32_ulp_diff(ks[b, hk, :n].cpu().numpy(), L.k_state).max() <= 1, lvl
            np.testing.assert_allclose(F[b, hk, :n].cpu().numpy(), L.F, rtol=1e-4, atol=0)


@pytest.mark.parametrize("name,T,B,h", [
    ("batched-decode-128k", 16384 + 64 * 5, 2, 16),   # partial rotary: 32 of 128 dims
    ("tiny-decode-f32", 8192, None, 64),              # fp32 cache, every dim rotated
    ("deep-tree-16m", 70000, None, 8),                # positions up to 7e4, three levels
])
def test_rope_tree_build_parity(name, T, B, h):
    base = S.workload(name)
    w = S.scaled(base, T=T, B=B, n_centres=min(base.n_centres, 1024))
    g = rope_geometry(w, h)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    freq = rope_table(h)
    tree = Z.empty_tree(g)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_build_tree(g, K, T, Z.reference_block(qref, freq), tree, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_tree(w, g, K, qref, freq, tree, T, [(b, hk) for b in range(w.B) for hk in range(w.Hkv)][:4])


def test_rope_tree_differs_from_plain_and_append_equals_rebuild():
    w = S.scaled(S.workload("prefill-append-256k"), T=16384 - 100, n_new=1300, n_centres=512)
    h = 16
    g = rope_geometry(w, h)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    qb = Z.reference_block(qref, rope_table(h))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    t1 = Z.empty_tree(g); t1.zero_()
    Z.zha_build_tree(g, K, w.T, qb, t1, st)
    t = w.T
    for piece in (1, 63, 500, 736):
        kn, vn = S.new_tokens(w, C, piece, DEV, step=t)
        Z.zha_append(g, K, V, kn, vn, t, qb, t1, st)
        t += piece
    t2 = Z.empty_tree(g); t2.zero_()
    Z.zha_build_tree(g, K, t, qb, t2, st)
    plain = Z.empty_tree(g); plain.zero_()
    Z.zha_build_tree(dataclasses.replace(g, rope_pairs=0), K, t, qref, plain, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(t1, t2)
    assert not torch.equal(t1, plain)
    check_tree(w, g, K, qref, rope_table(h), t1, t, [(0, 0), (0, 1)])


@pytest.mark.parametrize("name,T,B,p,h", [
    ("batched-decode-128k", 32768 + 9, 2, 0.95, 16),
    ("long-decode-1m", 65536 + 64 * 7 + 63, 1, 0.95, 32),   # the new token completes a leaf
])
def test_rope_decode_parity(name, T, B, p, h):
    base = S.workload(name)
    w = S.scaled(base, T=T, B=B, n_centres=min(base.n_centres, 1024))
    g = rope_geometry(w, h)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    freq = rope_table(h)
    qb = Z.reference_block(qref, freq)
    k_new, v_new = S.new_tokens(w, C, 1, DEV)
    q = S.queries(w, C, 1, DEV)
    tree = Z.empty_tree(g); tree.zero_()
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_DECODE)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_build_tree(g, K, w.T, qb, tree, st)
    cap = Z.leaf_cap(g)
    ids = torch.full((w.B, 1, w.Hq, cap), -7, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(w.B, 1, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(w.B, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
    Z.zha_decode(g, q, k_new, v_new, K, V, w.T, qb, p, tree, ids, cnt, O, ws, st)
    # per-level kept sets of the same routing
    nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
    lc = torch.zeros(w.B, 1, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
    lids = torch.full((w.B, 1, w.Hq, max(nst, 1)), -1, dtype=torch.int32, device=DEV)
    ids2, cnt2 = torch.full_like(ids, -7), torch.zeros_like(cnt)
    pos = torch.full((w.B, 1), w.T, dtype=torch.int64, device=DEV)
    Z.zha_route(g, q, pos, p, tree, ids2, cnt2, Z.empty_workspace(g, 1, Z.ZHA_OP_ROUTE), st, lc, lids)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(cnt, cnt2)
    Kc, Vc = K.cpu(), V.cpu()
    qr = qref.double().cpu().numpy()
    qc = q.double().cpu().numpy()
    Oc = O.float().cpu().numpy()
    ids_c, cnt_c, lc_c, lids_c = ids.cpu().numpy(), cnt.cpu().numpy(), lc.cpu().numpy(), lids.cpu().numpy()
    f = freq.double().numpy()
    cmp = RouteCompare()
    errs = []
    for (b, hk) in [(b, hk) for b in range(w.B) for hk in range(w.Hkv)][:3]:
        otree = zo.build_tree(Kc[b, hk], w.T + 1, qr[hk], w.depth, route_storage=route_storage(w), inv_freq=f)
        for hh in range(hk * w.G, (hk + 1) * w.G):
            levels, off = {}, 0
            for l in range(2, w.depth + 1):
                n = int(lc_c[b, 0, hh, l - 1, 1])
                levels[l] = lids_c[b, 0, hh, off:off + n].astype(np.int64)
                off += Z.tree_level(g, l).n_cap
            leaves = ids_c[b, 0, hh, :cnt_c[b, 0, hh]].astype(np.int64)
            leaves = compare_route(qc[b, 0, hh], w.T, otree, p, levels, leaves, cmp, f"b{b} h{hh}")
            o, _ = zo.attention(qc[b, 0, hh], Kc[b, hk], Vc[b, hk], zo.index_set(leaves, w.T))
            errs.append(np.abs(Oc[b, 0, hh] - o))
    assert cmp.ok(), cmp.problems()
    assert errs
    e = np.stack(errs)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())
    print(f"rope {w.name} h={h}: {cmp.summary()}")
