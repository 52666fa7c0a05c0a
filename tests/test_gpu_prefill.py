"""GPU parity of the query-tile prefill attention (zha_prefill_attn, tcgen05 tensor cores).

Every query keeps its own index set I(q) = {0} u (keys of S_1(q)) u C_cur(q) ("ZHA summary"
page, Routing); the tile only shares the gather (arXiv 2610.42112, App. A-B, Table I).  The
bar is the attention one: bf16 outputs within max-abs 2e-2 and mean-abs 2e-3 of the
oracle's attention over the same lists, the log-sum-exp within 1e-3 relative.
"""
import dataclasses

import numpy as np
import pytest
import torch

import zha_synth as S
from oracle import zha_oracle as zo
from tests.zha_cases import RouteCompare, compare_route, geometry

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def Z():
    import hierarchical_sparse_attention_02_b200 as z
    z.load_library()
    return z


def _prefill(Z, w, p=0.95):
    """Cache of T keys + n_new appended causal queries, their routes, and both attention
    paths (per query and per tile) on the same lists."""
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    tree = Z.empty_tree(g)
    Z.zha_build_tree(g, K, w.T, qref, tree, st)
    kn, vn = S.new_tokens(w, C, w.n_new, DEV)
    Z.zha_append(g, K, V, kn, vn, w.T, qref, tree, st)
    Q = S.queries(w, C, w.n_new, DEV)
    pos = (w.T + torch.arange(w.n_new, device=DEV, dtype=torch.int64)).view(1, -1).repeat(w.B, 1).contiguous()
    cap = Z.leaf_cap(g)
    ids = torch.full((w.B, w.n_new, w.Hq, cap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(w.B, w.n_new, w.Hq, dtype=torch.int32, device=DEV)
    nst = sum(Z.tree_level(g, l).n_cap for l in range(2, w.depth + 1))
    lcnt = torch.zeros(w.B, w.n_new, w.Hq, w.depth, 2, dtype=torch.int32, device=DEV)
    lids = torch.full((w.B, w.n_new, w.Hq, max(nst, 1)), -1, dtype=torch.int32, device=DEV)
    ws = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_ROUTE)
    Z.zha_route(g, Q, pos, p, tree, ids, cnt, ws, st, lcnt, lids)
    O1 = torch.empty(w.B, w.n_new, w.Hq, w.d, dtype=g.dtype, device=DEV)
    O2 = torch.empty_like(O1)
    l2 = torch.empty(w.B, w.n_new, w.Hq, dtype=torch.float32, device=DEV)
    wa = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_ATTN)
    Z.zha_sparse_attn(g, Q, K, V, pos, ids, cnt, O1, wa, st)
    wp = Z.empty_workspace(g, w.n_new, Z.ZHA_OP_PREFILL)
    Z.zha_prefill_attn(g, Q, K, V, pos, ids, cnt, O2, wp, st, lse=l2)
    torch.cuda.synchronize()
    assert st.item() == 0
    return dict(g=g, K=K, V=V, Q=Q, qref=qref, pos=pos, ids=ids, cnt=cnt, lcnt=lcnt, lids=lids, O1=O1, O2=O2,
                lse=l2)


@pytest.mark.parametrize("name,T,n_new,B", [
    ("prefill-append-256k", 20000, 512, 1),        # 32 tiles of 16 queries per KV head
    ("prefill-append-256k", 9000 + 37, 300, 2),    # a ragged last tile (300 = 18 * 16 + 12), two sequences
])
def test_prefill_tiles_match_the_oracle(Z, name, T, n_new, B):
    w = S.scaled(S.workload(name), T=T, n_new=n_new, B=B, n_centres=512)
    r = _prefill(Z, w)
    O1, O2 = r["O1"].float(), r["O2"].float()
    # the two GPU paths on the same lists
    d = (O1 - O2).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3, (d.max().item(), d.mean().item())
    # the oracle, routes compared level by level, outputs over the GPU's lists
    Kc, Vc = r["K"].cpu(), r["V"].cpu()
    qc = r["Q"].double().cpu().numpy()
    qr = r["qref"].double().cpu().numpy()
    g = r["g"]
    cmp = RouteCompare()
    errs = []
    rng = np.random.default_rng(5)
    for b in range(w.B):
        trees = {hk: zo.build_tree(Kc[b, hk], w.T + w.n_new, qr[hk], w.depth) for hk in range(w.Hkv)}
        for qi in sorted(set(rng.integers(0, w.n_new, 10).tolist()) | {0, 15, 16, w.n_new - 1}):
            t = w.T + qi
            for h in range(w.Hq):
                hk = h // w.G
                off, lv = 0, {}
                for l in range(2, w.depth + 1):
                    n = int(r["lcnt"][b, qi, h, l - 1, 1])
                    lv[l] = r["lids"][b, qi, h, off:off + n].cpu().numpy().astype(np.int64)
                    off += Z.tree_level(g, l).n_cap
                got = r["ids"][b, qi, h, :int(r["cnt"][b, qi, h])].cpu().numpy().astype(np.int64)
                leaves = compare_route(qc[b, qi, h], t, trees[hk], 0.95, lv, got, cmp, f"b{b} q{qi} h{h}")
                o, lse = zo.attention(qc[b, qi, h], Kc[b, hk], Vc[b, hk], zo.index_set(leaves, t))
                errs.append(np.abs(O2[b, qi, h].cpu().numpy() - o))
                assert abs(r["lse"][b, qi, h].item() - lse) <= 1e-3 * max(1.0, abs(lse))
    assert cmp.ok(), cmp.problems()
    e = np.stack(errs)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())
    print(f"prefill tiles {w.name} B={w.B}: {cmp.summary()}; max err {e.max():.2e}")


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (8, 8), (12, 4), (14, 2)])
def test_prefill_tiles_on_made_up_lists(Z, Hq, Hkv):
    """Random ascending leaf lists (empty ones, chunk 0 in or out), scattered positions
    (several own chunks per tile, a query at position 0), and group sizes G = 8, 1, 3, 7
    (tiles of 16, 128, 42 and 18 queries; the last two leave padding rows)."""
    base = S.workload("prefill-append-256k")
    w = dataclasses.replace(S.scaled(base, T=6000, n_new=1, B=1, n_centres=64), Hq=Hq, Hkv=Hkv)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    nq = 150
    Q = S.queries(w, C, nq, DEV)
    rng = np.random.default_rng(Hq * 100 + Hkv)
    pos_np = np.sort(rng.integers(0, w.T, nq))
    pos_np[0] = 0
    pos_np[-1] = w.T - 1
    cap = Z.leaf_cap(g)
    ids = np.full((1, nq, w.Hq, cap), -1, np.int32)
    cnt = np.zeros((1, nq, w.Hq), np.int32)
    for qi in range(nq):
        nvis = int(pos_np[qi]) // 64
        for h in range(w.Hq):
            k = int(rng.integers(0, nvis + 1)) if rng.random() < 0.9 else 0
            sel = np.sort(rng.choice(nvis, size=k, replace=False)) if k else np.zeros(0, int)
            ids[0, qi, h, :k] = sel
            cnt[0, qi, h] = k
    pos = torch.from_numpy(pos_np).view(1, -1).to(DEV)
    ids_d, cnt_d = torch.from_numpy(ids).to(DEV), torch.from_numpy(cnt).to(DEV)
    O = torch.empty(1, nq, w.Hq, w.d, dtype=g.dtype, device=DEV)
    lse = torch.empty(1, nq, w.Hq, dtype=torch.float32, device=DEV)
    ws = Z.empty_workspace(g, nq, Z.ZHA_OP_PREFILL)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Z.zha_prefill_attn(g, Q, K, V, pos, ids_d, cnt_d, O, ws, st, lse=lse)
    torch.cuda.synchronize()
    assert st.item() == 0
    Kc, Vc, qc = K.cpu(), V.cpu(), Q.double().cpu().numpy()
    errs = []
    for qi in range(nq):
        for h in range(w.Hq):
            idx = zo.index_set(ids[0, qi, h, :cnt[0, qi, h]], int(pos_np[qi]))
            o, l = zo.attention(qc[0, qi, h], Kc[0, h // w.G], Vc[0, h // w.G], idx)
            errs.append(np.abs(O[0, qi, h].float().cpu().numpy() - o))
            assert abs(lse[0, qi, h].item() - l) <= 1e-3 * max(1.0, abs(l)), (qi, h)
    e = np.stack(errs)
    assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())


def test_prefill_rejections_and_device_status(Z):
    w = S.scaled(S.workload("prefill-append-256k"), T=4096, n_new=1, B=1, n_centres=64)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    Q = S.queries(w, C, 20, DEV)
    cap = Z.leaf_cap(g)
    ids = torch.full((1, 20, w.Hq, cap), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros(1, 20, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(1, 20, w.Hq, w.d, dtype=g.dtype, device=DEV)
    ws = Z.empty_workspace(g, 20, Z.ZHA_OP_PREFILL)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    # a position beyond the cache: reported on the device, that query's rows untouched
    pos = torch.arange(20, dtype=torch.int64, device=DEV).view(1, -1) + 100
    pos[0, 7] = g.t_cap + 3
    Z.zha_prefill_attn(g, Q, K, V, pos.contiguous(), ids, cnt, O, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 1                                  # ZHA_ERR_INVALID_ARG
    # a leaf id at or past the query's own chunk
    st.zero_()
    pos = torch.full((1, 20), 1000, dtype=torch.int64, device=DEV)
    ids[0, 3, 0, 0] = 1000 // 64
    cnt[0, 3, 0] = 1
    Z.zha_prefill_attn(g, Q, K, V, pos, ids, cnt, O, ws, st)
    torch.cuda.synchronize()
    assert st.item() == 1
    # fp32 caches are not served by the tensor-core tile path
    g32 = geometry(S.scaled(S.workload("tiny-decode-f32"), T=4096))
    with pytest.raises(Z.ZhaError):
        Z.zha_prefill_attn(g32, Q, K, V, pos, ids, cnt, O, ws, st)
