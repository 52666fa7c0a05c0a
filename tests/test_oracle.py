"""Pins of the CPU oracle against facts fixed by the method and by mathematics.

Each test checks the oracle against something other than itself: a closed
form derived on paper (tests/golden), an independent identity (convexity lower
bound, entropy, gradient, entropy chain rule), brute-force enumeration, or a
textbook library routine.  They are chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, an
off-by-one in expansion or in the index set) makes at least one of them fail.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import zha_oracle as zo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")
LN = {"ln1": 0.0, "ln2": math.log(2), "ln3": math.log(3), "ln4": math.log(4), "ln10": math.log(10)}


def _ev(x):
    """Evaluate the tiny closed-form strings of the golden file."""
    if isinstance(x, (int, float)):
        return float(x)
    if x in LN:
        return LN[x]
    if x == "ln3/2":
        return math.log(3) / 2
    # forms "lnA - c*lnB" / "lnA - lnB"
    a, b = [s.strip() for s in x.split("-")]
    c, lb = b.split("*") if "*" in b else ("1", b)
    return LN[a] - float(c) * LN[lb]


@pytest.fixture(scope="module")
def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _clustered(T, d, n_centres, seed):
    rng = np.random.default_rng(seed)
    C = rng.standard_normal((n_centres, d))
    K = C[rng.integers(0, n_centres, T)] + 0.3 * rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    return C, K, V


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------


def test_round_bf16_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(zo.round_bf16(x.astype(np.float64)), ref)


def test_round_bf16_ties_to_even_and_no_double_rounding():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties to the even mantissa (1.0)
    assert zo.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 lies halfway between 1+2^-7 and 1+2^-6: ties to even (1+2^-6)
    assert zo.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    # just above the tie must round up; going through fp32 first would lose this
    x = 1 + 2 ** -8 + 2 ** -40
    assert zo.round_bf16(np.array([x]))[0] == 1 + 2 ** -7
    assert zo.round_bf16(np.array([-x]))[0] == -(1 + 2 ** -7)


# ---------------------------------------------------------------------------
# leaf summary
# ---------------------------------------------------------------------------


def test_leaf_closed_form(golden):
    g = golden["leaf_two_keys"]
    K = np.array(g["keys"], float)
    qref = np.array([[_ev(v) for v in row] for row in g["qref"]])
    k_hat, F, b_hat = zo.leaf_summary(K, qref, 1 / math.sqrt(g["d"]))
    assert F[0] == pytest.approx(_ev(g["F"]), abs=1e-14)
    np.testing.assert_allclose(k_hat[0], g["k_hat"], atol=1e-14)
    assert b_hat[0] == pytest.approx(_ev(g["b_hat"]), abs=1e-14)
    lvl = zo.Level(span=2, k_route=k_hat[None], b_hat=b_hat[None], F=F[None], k_state=k_hat[None])
    s0 = zo.node_scores(np.zeros(g["d"]), lvl, np.array([0]), 0.5)[0]
    assert s0 == pytest.approx(_ev(g["score_at_zero_query"]), abs=1e-14)
    assert zo.chunk_lse(np.zeros(g["d"]), K, 0.5) == pytest.approx(_ev(g["lse_at_zero_query"]), abs=1e-14)


@pytest.mark.parametrize("d", [8, 128])
def test_leaf_tangent_is_lower_bound_and_exact_at_reference(d):
    _, K, _ = _clustered(64, d, 16, 1)
    rng = np.random.default_rng(2)
    qref = rng.standard_normal((4, d)) / math.sqrt(d)
    scale = 1 / math.sqrt(d)
    k_hat, F, b_hat = zo.leaf_summary(K, qref, scale)
    lvl = zo.Level(64, k_hat[None], b_hat[None], F[None], k_hat[None])
    # convexity: every tangent lies below F_C, so does their max
    for _ in range(200):
        q = 2 * rng.standard_normal(d)
        assert zo.node_scores(q, lvl, np.array([0]), scale)[0] <= zo.chunk_lse(q, K, scale) + 1e-12
    # at each reference query the max of tangents touches F_C
    for r in range(4):
        s = zo.node_scores(qref[r], lvl, np.array([0]), scale)[0]
        assert s == pytest.approx(zo.chunk_lse(qref[r], K, scale), abs=1e-12)


@pytest.mark.parametrize("d", [8, 128])
def test_leaf_bias_is_entropy_and_k_hat_is_gradient(d):
    _, K, _ = _clustered(64, d, 8, 3)
    rng = np.random.default_rng(4)
    qref = 3 * rng.standard_normal((3, d)) / math.sqrt(d)
    scale = 1 / math.sqrt(d)
    k_hat, F, b_hat = zo.leaf_summary(K, qref, scale)
    for r in range(3):
        z = K @ qref[r] * scale
        a = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
        assert b_hat[r] == pytest.approx(-(a * np.log(a)).sum(), abs=1e-12)
        assert 0 <= b_hat[r] <= math.log(64) + 1e-12
        # central differences of F_C at q_hat_r give k_hat_r * scale
        h = 1e-5
        grad = np.array([(zo.chunk_lse(qref[r] + h * e, K, scale) - zo.chunk_lse(qref[r] - h * e, K, scale)) / (2 * h)
                         for e in np.eye(d)])
        np.testing.assert_allclose(grad, k_hat[r] * scale, atol=1e-8)


def test_leaf_special_cases():
    d = 16
    scale = 1 / math.sqrt(d)
    rng = np.random.default_rng(5)
    k = rng.standard_normal(d)
    Kc = np.tile(k, (64, 1))
    qref = rng.standard_normal((2, d))
    k_hat, F, b_hat = zo.leaf_summary(Kc, qref, scale)
    np.testing.assert_allclose(k_hat, np.tile(k, (2, 1)), atol=1e-13)
    np.testing.assert_allclose(b_hat, math.log(64), atol=1e-13)
    lvl = zo.Level(64, k_hat[None], b_hat[None], F[None], k_hat[None])
    q = rng.standard_normal(d)
    assert zo.node_scores(q, lvl, np.array([0]), scale)[0] == pytest.approx(zo.chunk_lse(q, Kc, scale), abs=1e-12)
    # a zero reference query weighs all keys equally
    _, K, _ = _clustered(64, d, 4, 6)
    k_hat, F, b_hat = zo.leaf_summary(K, np.zeros((1, d)), scale)
    np.testing.assert_allclose(k_hat[0], K.mean(0), atol=1e-13)
    assert b_hat[0] == pytest.approx(math.log(64), abs=1e-13)


# ---------------------------------------------------------------------------
# parent merge
# ---------------------------------------------------------------------------


def test_merge_closed_form(golden):
    g = golden["merge_two_children"]
    qref = np.array([[_ev(v) for v in row] for row in g["qref"]])
    scale = 1 / math.sqrt(g["d"])
    kids = [zo.leaf_summary(np.array(c, float), qref, scale) for c in g["children"]]
    F_c = np.stack([k[1] for k in kids])
    k_c = np.stack([k[0] for k in kids])
    k_hat, F, b_hat = zo.merge_summaries(F_c, k_c, qref, scale)
    assert F[0] == pytest.approx(_ev(g["F"]), abs=1e-14)
    np.testing.assert_allclose(k_hat[0], g["k_hat"], atol=1e-14)
    assert b_hat[0] == pytest.approx(_ev(g["b_hat"]), abs=1e-14)


@pytest.mark.parametrize("d", [8, 128])
def test_merged_tree_equals_leaf_formula_over_span(d):
    T = 64 * 16 * 16 * 2
    _, K, _ = _clustered(T, d, 32, 7)
    rng = np.random.default_rng(8)
    qref = 4 * rng.standard_normal((4, d)) / math.sqrt(d)
    scale = 1 / math.sqrt(d)
    tree = zo.build_tree(K, T, qref, depth=3, route_storage="f64", state_storage="f64")
    assert [lv.n for lv in tree.levels] == [T // 64, T // 1024, T // 16384]
    for lvl in (2, 3):
        span = tree.span(lvl)
        for i in range(tree.levels[lvl - 1].n):
            k_hat, F, b_hat = zo.leaf_summary(K[i * span:(i + 1) * span], qref, scale)
            L = tree.levels[lvl - 1]
            np.testing.assert_allclose(L.F[i], F, rtol=0, atol=1e-12)
            np.testing.assert_allclose(L.k_state[i], k_hat, rtol=0, atol=1e-12)
            np.testing.assert_allclose(L.b_hat[i], b_hat, rtol=0, atol=1e-11)


TREE_FREQ = [1.0, 0.37, 0.05]     # partial rotary frequencies for the rotated-tree cases


@pytest.mark.parametrize("d", [8, 128])
@pytest.mark.parametrize("rotary", [False, True])
def test_build_tree_nodes_equal_the_per_node_formulas(d, rotary):
    """Every node of build_tree (its batched level passes) equals the one-node formulas:
    a level-1 node is ``leaf_summary`` over its own keys at its own reference queries, a
    level-l node ``merge_summaries`` over its stored children.  The batched passes are
    pinned to the one-node functions, which the closed forms and identities pin."""
    leaf, branch, depth = 8, 4, 3
    T = leaf * branch ** 2 * 3 + leaf * 5 + 3              # ragged: orphan leaves and a partial chunk
    _, K, _ = _clustered(T, d, 12, 31 + d)
    rng = np.random.default_rng(32)
    qref = 3 * rng.standard_normal((4, d)) / math.sqrt(d)
    scale = 1 / math.sqrt(d)
    freq = TREE_FREQ if rotary else None
    tree = zo.build_tree(K, T, qref, depth, leaf=leaf, branch=branch, route_storage="f64",
                         state_storage="f64", block=7, inv_freq=freq)
    assert [lv.n for lv in tree.levels] == [T // leaf, T // (leaf * branch), T // (leaf * branch ** 2)]

    def refs(level, i):
        if not rotary:
            return qref
        return zo.rope(qref, zo.node_anchor(i, tree.span(level)), freq)

    L1 = tree.levels[0]
    for i in range(L1.n):
        k_hat, F, b_hat = zo.leaf_summary(K[i * leaf:(i + 1) * leaf], refs(1, i), scale)
        np.testing.assert_allclose(L1.F[i], F, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L1.k_state[i], k_hat, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L1.k_route[i], k_hat, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L1.b_hat[i], b_hat, rtol=0, atol=1e-12)
    for lvl in range(2, depth + 1):
        child, lv = tree.levels[lvl - 2], tree.levels[lvl - 1]
        for i in range(lv.n):
            ids = np.arange(i * branch, (i + 1) * branch)
            q_c = np.stack([refs(lvl - 1, c) for c in ids]) if rotary else None
            k_hat, F, b_hat = zo.merge_summaries(child.F[ids], child.k_state[ids], refs(lvl, i), scale,
                                                 q_child=q_c)
            np.testing.assert_allclose(lv.F[i], F, rtol=0, atol=1e-13)
            np.testing.assert_allclose(lv.k_state[i], k_hat, rtol=0, atol=1e-13)
            np.testing.assert_allclose(lv.b_hat[i], b_hat, rtol=0, atol=1e-12)


def test_merge_entropy_chain_rule():
    d = 32
    _, K, _ = _clustered(64 * 16, d, 16, 9)
    rng = np.random.default_rng(10)
    qref = 2 * rng.standard_normal((3, d)) / math.sqrt(d)
    scale = 1 / math.sqrt(d)
    kids = [zo.leaf_summary(K[c * 64:(c + 1) * 64], qref, scale) for c in range(16)]
    F_c = np.stack([k[1] for k in kids])
    b_c = np.stack([k[2] for k in kids])
    _, F, b_hat = zo.merge_summaries(F_c, np.stack([k[0] for k in kids]), qref, scale)
    w = np.exp(F_c - F[None])
    np.testing.assert_allclose(b_hat, (w * b_c).sum(0) - (w * np.log(w)).sum(0), atol=1e-12)


def test_stored_tree_rounds_where_stored():
    d = 128
    T = 64 * 16
    _, K, _ = _clustered(T, d, 16, 11)
    qref = np.random.default_rng(12).standard_normal((4, d)) / math.sqrt(d)
    t = zo.build_tree(K, T, qref, depth=2, route_storage="bf16", state_storage="f32")
    L1 = t.levels[0]
    np.testing.assert_array_equal(L1.k_route, zo.round_bf16(L1.k_route))
    np.testing.assert_array_equal(L1.k_state, L1.k_state.astype(np.float32))
    np.testing.assert_array_equal(L1.F, L1.F.astype(np.float32))
    exact = zo.build_tree(K, T, qref, depth=2, route_storage="f64", state_storage="f64")
    np.testing.assert_allclose(t.levels[1].k_state, exact.levels[1].k_state, rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------------------
# top-p selection
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("case", ["top_p_ties", "top_p_exact_boundary"])
def test_top_p_closed_form_with_ties(golden, case):
    g = golden[case]
    sel = zo.top_p(np.array([_ev(s) for s in g["scores"]]), np.array(g["ids"]), g["p"])
    assert sel.m == g["m"]
    assert sel.ids.tolist() == g["selected"]


def _brute_min_subset(scores, p):
    """Smallest cardinality of a subset with softmax mass >= p, and the max-mass such subset."""
    e = np.exp(scores - scores.max())
    pi = e / e.sum()
    n = len(scores)
    for k in range(1, n + 1):
        best, best_mass = None, -1.0
        for sub in itertools.combinations(range(n), k):
            mass = pi[list(sub)].sum()
            if mass > best_mass:
                best, best_mass = sub, mass
        if best_mass >= p:
            return k, set(best)
    return n, set(range(n))


@pytest.mark.parametrize("seed", range(25))
def test_top_p_is_minimal_by_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 11))
    scores = rng.standard_normal(n) * rng.uniform(0.1, 3)
    ids = rng.permutation(1000)[:n]
    p = float(rng.uniform(0.05, 0.99))
    sel = zo.top_p(scores, ids, p)
    k, best = _brute_min_subset(scores, p)
    assert sel.m == k
    assert set(sel.ids.tolist()) == {int(ids[i]) for i in best}
    # the cutoff straddles p
    order = np.lexsort((ids, -scores))
    e = np.exp(scores[order] - scores.max())
    cum = np.cumsum(e / e.sum())
    assert cum[sel.m - 1] >= p and (sel.m == 1 or cum[sel.m - 2] < p)


def test_top_p_one_keeps_all():
    s = np.array([3.0, -50.0, -800.0, 0.5])
    assert zo.top_p(s, np.arange(4), 1.0).ids.tolist() == [0, 1, 2, 3]


# ---------------------------------------------------------------------------
# routing, index set and attention
# ---------------------------------------------------------------------------


def test_index_set_closed_forms(golden):
    g = golden["index_set"]
    for c in g["cases"]:
        want = np.concatenate([np.arange(a, b + 1) for a, b in c["ranges"]])
        np.testing.assert_array_equal(zo.index_set(c["leaves"], c["t"], g["leaf"]), want)


def test_expansion_with_orphans_hand_example():
    # leaf=4, branch=4: t=73 -> V=72: 18 visible leaves, 4 visible level-2 nodes, 1 level-3 node
    d = 8
    _, K, _ = _clustered(80, d, 4, 13)
    qref = np.random.default_rng(14).standard_normal((2, d)) / math.sqrt(d)
    tree = zo.build_tree(K, 80, qref, depth=4, leaf=4, branch=4, route_storage="f64")
    r = zo.route(np.ones(d), 73, tree, 1.0)
    assert r.top == 3
    assert r.cand[3].tolist() == [0]
    assert r.cand[2].tolist() == [0, 1, 2, 3]
    assert r.cand[1].tolist() == list(range(16)) + [16, 17]
    # t=40 -> V=40: 10 leaves, 2 level-2 nodes, no level-3 node: level 2 is the top
    r = zo.route(np.ones(d), 40, tree, 1.0)
    assert r.top == 2 and r.cand[2].tolist() == [0, 1]
    assert r.cand[1].tolist() == list(range(8)) + [8, 9]
    # t=3: nothing visible
    r = zo.route(np.ones(d), 3, tree, 1.0)
    assert r.top == 0 and len(r.leaves) == 0


def _torch_softmax_attention(q, K, V):
    z = torch.from_numpy(K) @ torch.from_numpy(q) / math.sqrt(q.shape[0])
    return (torch.softmax(z, 0) @ torch.from_numpy(V)).numpy()


@pytest.mark.parametrize("d,T,t", [(8, 4096, 4095), (128, 4096, 3000), (128, 1024 * 3 + 70, 1024 * 3 + 69)])
def test_p_one_routing_reproduces_dense_attention(d, T, t):
    C, K, V = _clustered(T, d, 64, 15)
    qref = np.random.default_rng(16).standard_normal((4, d)) / math.sqrt(d)
    tree = zo.build_tree(K, T, qref, depth=3, route_storage="bf16")
    q = 2 * C[5] + 0.3 * np.random.default_rng(17).standard_normal(d)
    r, o, _ = zo.decode_head(q, K, V, t, tree, 1.0)
    assert len(r.leaves) == t // 64
    np.testing.assert_array_equal(zo.index_set(r.leaves, t), np.arange(t + 1))
    np.testing.assert_allclose(o, _torch_softmax_attention(q, K[:t + 1], V[:t + 1]), atol=1e-12)


@pytest.mark.parametrize("p", [0.5, 0.9, 0.99])
def test_top_p_decomposition_eq1(p):
    d, T = 128, 4096
    C, K, V = _clustered(T, d, 64, 18)
    qref = np.random.default_rng(19).standard_normal((4, d)) / math.sqrt(d)
    tree = zo.build_tree(K, T, qref, depth=2)
    q = 2 * C[3] + 0.3 * np.random.default_rng(20).standard_normal(d)
    t = T - 1
    r = zo.route(q, t, tree, p)
    S = zo.index_set(r.leaves, t)
    Sbar = np.setdiff1d(np.arange(t + 1), S)
    z = K[:t + 1] @ q / math.sqrt(d)
    a = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    P_S = a[S].sum()
    full = _torch_softmax_attention(q, K[:t + 1], V[:t + 1])
    oS, _ = zo.attention(q, K, V, S)
    oSbar = _torch_softmax_attention(q, K[Sbar], V[Sbar]) if len(Sbar) else np.zeros(d)
    np.testing.assert_allclose(full, P_S * oS + (1 - P_S) * oSbar, atol=1e-12)


def test_whole_route_levels_by_brute_force():
    # small geometry (leaf 4, branch 4) so that every level has <= 16 candidates
    d = 8
    T = 64
    C, K, V = _clustered(T, d, 4, 21)
    rng = np.random.default_rng(22)
    qref = rng.standard_normal((2, d)) / math.sqrt(d)
    tree = zo.build_tree(K, T, qref, depth=3, leaf=4, branch=4, route_storage="f64")
    for trial in range(20):
        q = 2 * C[trial % 4] + 0.3 * rng.standard_normal(d)
        p = float(rng.uniform(0.3, 0.95))
        r = zo.route(q, 63, tree, p)
        for lvl, cand in r.cand.items():
            s = zo.node_scores(q, tree.levels[lvl - 1], cand, 1 / math.sqrt(d))
            k, best = _brute_min_subset(s, p)
            assert r.sel[lvl].m == k
            assert set(r.sel[lvl].ids.tolist()) == {int(cand[i]) for i in best}


def test_flat_scores_are_exact_chunk_lse():
    d, T = 16, 64 * 5 + 10
    _, K, _ = _clustered(T, d, 4, 23)
    q = np.random.default_rng(24).standard_normal(d)
    s = zo.flat_scores(q, K, T - 1)
    assert len(s) == 5
    for c in range(5):
        brute = math.log(sum(math.exp(float(K[j] @ q) / 4.0) for j in range(c * 64, (c + 1) * 64)))
        assert s[c] == pytest.approx(brute, abs=1e-12)
