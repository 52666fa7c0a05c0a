"""The parity harness itself, on the CPU: how a GPU route that differs from the oracle's is
judged (tests/zha_cases.py ``compare_route`` / ``near_cutoff_valid``) and the oracle's
``impose`` hook that continues a route from a given kept set.  Every GPU set below is
made up on the host."""
import math

import numpy as np
import pytest

from oracle import zha_oracle as zo
from tests.zha_cases import NEAR_CUTOFF, RouteCompare, compare_route, near_cutoff_valid

D = 8


def _tree(T=256, seed=3, depth=2):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((T, D))
    qref = rng.standard_normal((2, D)) / math.sqrt(D)
    return zo.build_tree(K, T, qref, depth=depth, leaf=4, branch=4, route_storage="f64", state_storage="f64")


def _gpu_sets(r):
    return {l: r.kept[l] for l in r.kept if l > 1}, r.kept[1]


def test_impose_expands_the_imposed_set():
    tree = _tree()
    q = np.random.default_rng(4).standard_normal(D)
    r = zo.route(q, 255, tree, 0.9)
    assert np.array_equal(zo.route(q, 255, tree, 0.9, impose={2: r.sel[2].ids}).leaves, r.leaves)
    pick = np.array([1, 7, 12])
    r2 = zo.route(q, 255, tree, 0.9, impose={2: pick})
    # t = 255: leaves 0..62 and level-2 nodes 0..14 are visible, so leaves 60..62 are orphans
    want = np.concatenate([(pick[:, None] * 4 + np.arange(4)).ravel(), [60, 61, 62]])
    assert np.array_equal(r2.cand[1], want)
    assert np.array_equal(r2.kept[2], pick)
    assert set(r2.leaves) <= set(want)
    with pytest.raises(ValueError):
        zo.route(q, 255, tree, 0.9, impose={2: np.array([3, 3])})
    with pytest.raises(ValueError):
        zo.route(q, 255, tree, 0.9, impose={2: np.array([64])})


def test_identical_routes_are_exact():
    tree = _tree()
    cmp = RouteCompare()
    for s in range(6):
        q = np.random.default_rng(10 + s).standard_normal(D)
        r = zo.route(q, 255, tree, 0.9)
        lv, leaves = _gpu_sets(r)
        assert np.array_equal(compare_route(q, 255, tree, 0.9, lv, leaves, cmp, "h"), r.leaves)
    assert cmp.exact == 6 and cmp.near_cutoff == 0 and cmp.ok()


def _near_cutoff_case():
    """A one-level tree (the candidates do not depend on p), a query and a p placed just
    above the oracle's cumulative mass of its m best leaves, so that keeping those m (one
    fewer than the oracle) is within NEAR_CUTOFF."""
    tree = _tree(depth=1)
    q = np.random.default_rng(21).standard_normal(D)
    r = zo.route(q, 255, tree, 0.9)
    cand = r.cand[1]
    s = zo.node_scores(q, tree.levels[0], cand, 1 / math.sqrt(D))
    order = np.lexsort((cand, -s))
    pi = np.exp(s[order] - s[order][0])
    pi /= pi.sum()
    cum = np.cumsum(pi)
    m = len(cand) // 2
    p = float(cum[m - 1]) + NEAR_CUTOFF / 4                      # the oracle keeps m + 1
    return tree, q, p, cand[order], m


def test_near_cutoff_difference_is_counted_and_the_output_uses_the_gpu_list():
    tree, q, p, ranked, m = _near_cutoff_case()
    r = zo.route(q, 255, tree, p)
    assert r.sel[1].m == m + 1
    lv, _ = _gpu_sets(r)
    gpu = np.sort(ranked[:m])                                     # one fewer: mass p - NEAR_CUTOFF / 4
    cmp = RouteCompare()
    leaves = compare_route(q, 255, tree, p, lv, gpu, cmp, "h")
    assert cmp.near_cutoff == 1 and cmp.exact == 0 and not cmp.mismatched
    assert np.array_equal(leaves, gpu)
    assert cmp.ok()                                               # one excused head is allowed


def test_wrong_sets_fail():
    tree, q, p, ranked, m = _near_cutoff_case()
    r = zo.route(q, 255, tree, p)
    lv, _ = _gpu_sets(r)
    for bad in (np.sort(ranked[:m - 3]),                         # several short: mass far below p
                np.sort(ranked[:m + 4]),                         # not minimal
                np.sort(np.concatenate([ranked[:m], ranked[-1:]])),   # the worst candidate kept
                np.sort(ranked[:m + 1])[::-1]):                  # not ascending
        cmp = RouteCompare()
        compare_route(q, 255, tree, p, lv, bad, cmp, "h")
        assert not cmp.ok(), bad


def test_too_many_excused_heads_fail():
    cmp = RouteCompare(heads=64, near_cutoff=3)
    assert cmp.excused_limit() == 2 and not cmp.ok()
    assert RouteCompare(heads=64, near_cutoff=2).ok()


def test_near_cutoff_valid_rules():
    s = np.log(np.array([0.5, 0.3, 0.15, 0.05]))
    c = np.arange(4)
    assert near_cutoff_valid(s, c, np.array([0, 1, 2]), 0.95) == ""
    assert near_cutoff_valid(s, c, np.array([0, 1]), 0.95) != ""          # mass 0.8
    assert near_cutoff_valid(s, c, np.array([0, 1, 2, 3]), 0.9) != ""     # not minimal
    assert near_cutoff_valid(s, c, np.array([0, 1]), 0.8 + NEAR_CUTOFF / 2) == ""
    assert near_cutoff_valid(s, c, np.array([0, 2, 3]), 0.5) != ""        # 1 outscores 2 and 3
    assert near_cutoff_valid(s, c, np.array([0, 1, 2]), 1.0) != ""        # p = 1 keeps all
    assert near_cutoff_valid(s, c, np.array([0, 1]), None, k=2) == ""
    assert near_cutoff_valid(s, c, np.array([0, 2]), None, k=2) != ""
    tie = np.array([1.0, 1.0 + NEAR_CUTOFF / 2, 0.0])
    assert near_cutoff_valid(tie, np.arange(3), np.array([0]), None, k=1) == ""   # a near tie may swap
    far = np.array([1.0, 1.01, 0.0])                                              # mass gap ~ 3.5e-3
    assert near_cutoff_valid(far, np.arange(3), np.array([0]), None, k=1) != ""
