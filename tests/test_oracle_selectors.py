"""Pins of the oracle's selector variants: the fixed-count selector (top-K, the budget
K of the roofline-model variables in arXiv 2610.42112 App. D, Table VI) and per-level
threshold schedules (constant p, §IV-A; p**(1/L), §VII "Asymptotic length scaling").

Each check compares the oracle with brute-force enumeration or with a closed form that
does not go through the routing loop (for instance: with p = 1 above the leaves, the
leaf selection is the top-p of every visible leaf chunk scored on its own).
"""
import itertools
import math

import numpy as np
import pytest

from oracle import zha_oracle as zo


def _clustered(T, d, n_centres, seed):
    rng = np.random.default_rng(seed)
    C = rng.standard_normal((n_centres, d))
    K = C[rng.integers(0, n_centres, T)] + 0.3 * rng.standard_normal((T, d))
    return C, K


def _brute_top_k(scores, ids, k):
    """Of all subsets of size min(k, n), the one whose members, listed best first by
    (score desc, id asc), are elementwise first: found by enumerating every subset."""
    n = len(ids)
    m = min(k, n)
    best = None
    for sub in itertools.combinations(range(n), m):
        key = sorted((-scores[i], ids[i]) for i in sub)
        if best is None or key < best[0]:
            best = (key, sub)
    return sorted(int(ids[i]) for i in best[1]) if m > 0 else []


@pytest.mark.parametrize("seed", range(30))
def test_top_k_by_brute_force(seed):
    rng = np.random.default_rng(500 + seed)
    n = int(rng.integers(1, 10))
    scores = rng.standard_normal(n) * rng.uniform(0.1, 3)
    if seed % 3 == 0:
        scores = np.round(scores)                  # ties: the id decides
    ids = rng.permutation(1000)[:n]
    for k in range(0, n + 3):
        sel = zo.top_k(scores, ids, k)
        assert sel.m == min(k, n)
        assert sel.ids.tolist() == _brute_top_k(scores, ids, k)
        chosen = set(sel.ids.tolist())
        for i in range(n):                         # every kept candidate outranks every dropped one
            for j in range(n):
                if int(ids[i]) in chosen and int(ids[j]) not in chosen:
                    assert (scores[i], -ids[i]) > (scores[j], -ids[j])


def test_top_k_keeps_the_top_p_set_at_its_size():
    rng = np.random.default_rng(7)
    for _ in range(50):
        n = int(rng.integers(1, 40))
        s = rng.standard_normal(n) * 2
        ids = rng.permutation(5000)[:n]
        tp = zo.top_p(s, ids, float(rng.uniform(0.1, 0.99)))
        assert zo.top_k(s, ids, tp.m).ids.tolist() == tp.ids.tolist()


def test_p_root_schedule():
    for p in (0.5, 0.9, 0.95, 0.99):
        for L in range(1, 9):
            sched = zo.p_root_schedule(p, L)
            assert len(sched) == L
            assert math.prod(sched) == pytest.approx(p, rel=1e-14)
            assert all(x == sched[0] and p <= x <= 1.0 for x in sched)
    assert zo.p_root_schedule(0.9, 1) == [0.9]


def _tree(T=80, d=8, depth=4, seed=31):
    # leaf 4, branch 4: at t = 73 there are 18 visible leaves (16 under level-2 nodes,
    # 2 orphans), 4 visible level-2 nodes and one level-3 node
    C, K = _clustered(T, d, 4, seed)
    qref = np.random.default_rng(seed + 1).standard_normal((2, d)) / math.sqrt(d)
    return C, zo.build_tree(K, T, qref, depth=depth, leaf=4, branch=4, route_storage="f64")


def test_schedule_with_p_one_above_the_leaves_is_flat_top_p_over_leaf_summaries():
    C, tree = _tree()
    d = 8
    scale = 1 / math.sqrt(d)
    rng = np.random.default_rng(40)
    leaves = np.arange(18)
    for trial in range(20):
        q = 2 * C[trial % 4] + 0.3 * rng.standard_normal(d)
        p1 = float(rng.uniform(0.2, 0.95))
        r = zo.route(q, 73, tree, [p1, 1.0, 1.0, 1.0])
        want = zo.top_p(zo.node_scores(q, tree.levels[0], leaves, scale), leaves, p1)
        assert r.cand[1].tolist() == leaves.tolist()
        assert r.leaves.tolist() == want.ids.tolist()


def test_top_k_with_budgets_above_every_level_keeps_everything():
    C, tree = _tree()
    r = zo.route(np.ones(8), 73, tree, 0.5, k=10 ** 6)
    assert r.top == 3
    assert r.leaves.tolist() == list(range(18))


def test_top_k_at_the_leaves_only_is_the_k_best_visible_leaves():
    C, tree = _tree()
    d = 8
    scale = 1 / math.sqrt(d)
    rng = np.random.default_rng(41)
    for trial in range(10):
        q = 2 * C[trial % 4] + 0.3 * rng.standard_normal(d)
        k1 = int(rng.integers(1, 19))
        r = zo.route(q, 73, tree, 0.5, k=[k1, 99, 99, 99])
        s = zo.node_scores(q, tree.levels[0], np.arange(18), scale)
        assert r.leaves.tolist() == _brute_top_k(s, np.arange(18), k1)


@pytest.mark.parametrize("selector", ["schedule", "top_k"])
def test_whole_route_with_per_level_parameters_by_brute_force(selector):
    """Distinct parameters per level: each level's selection is checked by brute force
    with the parameter of that level (so an off-by-one in the level index fails)."""
    d, T = 8, 64
    C, K = _clustered(T, d, 4, 51)
    rng = np.random.default_rng(52)
    qref = rng.standard_normal((2, d)) / math.sqrt(d)
    tree = zo.build_tree(K, T, qref, depth=3, leaf=4, branch=4, route_storage="f64")
    scale = 1 / math.sqrt(d)
    for trial in range(20):
        q = 2 * C[trial % 4] + 0.3 * rng.standard_normal(d)
        if selector == "schedule":
            ps = [float(x) for x in rng.uniform(0.3, 0.97, 3)]
            r = zo.route(q, 63, tree, ps)
        else:
            ks = [int(x) for x in rng.integers(1, 6, 3)]
            r = zo.route(q, 63, tree, 0.5, k=ks)
        for lvl, cand in r.cand.items():
            s = zo.node_scores(q, tree.levels[lvl - 1], cand, scale)
            if selector == "schedule":
                e = np.exp(s - s.max())
                pi = e / e.sum()
                # smallest subset reaching the level's p, by enumeration
                m = next(k for k in range(1, len(s) + 1)
                         if max(pi[list(c)].sum() for c in itertools.combinations(range(len(s)), k))
                         >= ps[lvl - 1])
                assert r.sel[lvl].m == m
            else:
                assert r.sel[lvl].ids.tolist() == _brute_top_k(s, cand, ks[lvl - 1])
