"""Failure detection on the GPU without a fault: a bounded device wait that runs out.

zha_check_bounded_wait runs the attention rings' own bounded mbarrier wait on a barrier
that nothing completes.  The wait must give up within its limit, report ZHA_ERR_DEVICE
through the status word, stop the CTA's other waiting warp through the abort flag, and
leave the context usable: a decode step right after it runs clean and matches the oracle.
"""
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


@pytest.mark.parametrize("polls", [1 << 10, 1 << 16])
def test_bounded_wait_gives_up_and_the_context_stays_usable(Z, polls):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.full((4,), -1, dtype=torch.int64, device=DEV)
    Z.zha_check_bounded_wait(polls, st, out)
    torch.cuda.synchronize()
    assert st.item() == 5                                    # ZHA_ERR_DEVICE
    cyc0, cyc1, gave0, gave1 = out.cpu().tolist()
    assert gave0 == 1 and gave1 == 1
    assert cyc0 >= polls                                     # at least a cycle per poll
    # warp 1 has 64x the limit but returns on the abort flag shortly after warp 0 gives up
    assert cyc1 < 4 * cyc0 + 100000, (cyc0, cyc1)

    # the same context: one decode step, clean status, routes and outputs as the oracle's
    w = S.scaled(S.workload("batched-decode-128k"), T=4096 + 70, B=1, n_centres=128)
    g = geometry(w)
    C, K, V = S.clustered_kv(w, DEV)
    qref = S.reference_queries(w, DEV)
    kn, vn = S.new_tokens(w, C, 1, DEV)
    q = S.queries(w, C, 1, DEV)
    tree = Z.empty_tree(g)
    ws = Z.empty_workspace(g, 1, Z.ZHA_OP_DECODE)
    st2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    ids = torch.empty(1, 1, w.Hq, Z.leaf_cap(g), dtype=torch.int32, device=DEV)
    cnt = torch.empty(1, 1, w.Hq, dtype=torch.int32, device=DEV)
    O = torch.empty(1, 1, w.Hq, w.d, dtype=g.dtype, device=DEV)
    Z.zha_build_tree(g, K, w.T, qref, tree, st2)
    Z.zha_decode(g, q, kn, vn, K, V, w.T, qref, 0.95, tree, ids, cnt, O, ws, st2)
    torch.cuda.synchronize()
    assert st2.item() == 0
    Kc, Vc = K.cpu(), V.cpu()
    qc = q.double().cpu().numpy()
    cmp = RouteCompare()
    for hk in range(w.Hkv):
        t = zo.build_tree(Kc[0, hk], w.T + 1, qref[hk].double().cpu().numpy(), w.depth)
        for h in range(hk * w.G, (hk + 1) * w.G):
            got = ids[0, 0, h, :int(cnt[0, 0, h])].cpu().numpy().astype(np.int64)
            r = zo.route(qc[0, 0, h], w.T, t, 0.95)
            levels = {l: r.sel[l].ids for l in r.sel if l > 1}   # only the leaves are reported by decode
            leaves = compare_route(qc[0, 0, h], w.T, t, 0.95, levels, got, cmp, f"h{h}")
            o, _ = zo.attention(qc[0, 0, h], Kc[0, hk], Vc[0, hk], zo.index_set(leaves, w.T))
            assert np.abs(O[0, 0, h].float().cpu().numpy() - o).max() <= 2e-2
    assert cmp.ok(), cmp.problems()
