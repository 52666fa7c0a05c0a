"""Pins of the oracle's rotary-position variant of the tree (arXiv 2610.42112 §III-B: the
shared reference queries are rotated to the last position of each node's span, and a parent
moves each child's estimated log mass to its own rotated reference along the child's tangent
plane before merging).

What fixes the answer independently of the oracle's code:
  * the rotation is multiplication of the complex pairs (x_i + i x_{i+h}) by e^{i pos f_i}
    (checked with numpy complex arithmetic), and scores depend only on relative positions;
  * a leaf's tangent is exact at its own rotated reference (closed form, as without RoPE);
  * children whose keys are all equal have an affine log mass, so re-anchoring is exact and
    the parent must equal the leaf formula over its whole span at the parent's rotated
    reference (to rounding);
  * every node's tangent lies below the exact log mass of its span for every query
    (convexity, by induction over the levels), with rotation as without;
  * with no frequencies the tree is the plain one, bit for bit.
"""
import math

import numpy as np
import pytest

from oracle import zha_oracle as zo

D = 8
FREQ = [1.0, 0.37, 0.05]          # partial rotary: dims 0..5 rotate, 6..7 pass through


def test_rope_is_complex_multiplication():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, D))
    pos = np.array([0, 1, 7, 1000, 123456])
    h = len(FREQ)
    z = (x[:, :h] + 1j * x[:, h:2 * h]) * np.exp(1j * pos[:, None] * np.array(FREQ)[None, :])
    want = np.concatenate([z.real, z.imag, x[:, 2 * h:]], axis=1)
    np.testing.assert_allclose(zo.rope(x, pos, FREQ), want, rtol=0, atol=1e-12)
    # d = 2 with one frequency 1: a rotation by pos radians
    np.testing.assert_allclose(zo.rope(np.array([1.0, 0.0]), 0.5, [1.0]), [math.cos(0.5), math.sin(0.5)],
                               atol=1e-15)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(2)
    for _ in range(20):
        q, k = rng.standard_normal(D), rng.standard_normal(D)
        m, n = (int(v) for v in rng.integers(0, 10 ** 6, 2))
        a = zo.rope(q, m, FREQ) @ zo.rope(k, n, FREQ)
        b = zo.rope(q, m - n, FREQ) @ k
        assert a == pytest.approx(b, abs=1e-9)
        assert np.linalg.norm(zo.rope(q, m, FREQ)) == pytest.approx(np.linalg.norm(q), rel=1e-14)
    x = rng.standard_normal(D)
    np.testing.assert_array_equal(zo.rope(x, 0, FREQ), x)
    np.testing.assert_array_equal(zo.rope(x, 99, []), x)


def _keys(T, seed, const_block=1):
    """Clustered keys; with const_block > 1 every block of that many keys holds one key."""
    rng = np.random.default_rng(seed)
    C = rng.standard_normal((6, D))
    nb = T // const_block
    K = C[rng.integers(0, 6, nb)] + 0.3 * rng.standard_normal((nb, D))
    return np.repeat(K, const_block, axis=0)


def _qref(R=3, seed=9):
    return np.random.default_rng(seed).standard_normal((R, D))


def test_no_frequencies_is_the_plain_tree_bit_for_bit():
    K = _keys(256, 3)
    plain = zo.build_tree(K, 256, _qref(), depth=3, leaf=4, branch=4, route_storage="f64")
    rot0 = zo.build_tree(K, 256, _qref(), depth=3, leaf=4, branch=4, route_storage="f64", inv_freq=[])
    for a, b in zip(plain.levels, rot0.levels):
        for f in ("k_route", "b_hat", "F", "k_state"):
            np.testing.assert_array_equal(getattr(a, f), getattr(b, f))


def test_leaf_tangent_exact_at_its_rotated_reference():
    K = _keys(256, 4)
    qref = _qref()
    tree = zo.build_tree(K, 256, qref, depth=2, leaf=4, branch=4, route_storage="f64", state_storage="f64",
                         inv_freq=FREQ)
    scale = 1 / math.sqrt(D)
    lv = tree.levels[0]
    for i in range(lv.n):
        for r in range(qref.shape[0]):
            q = zo.rope(qref[r], 4 * i + 3, FREQ)          # the leaf's last key is at 4i + 3
            exact = zo.chunk_lse(q, K[4 * i:4 * i + 4], scale)
            assert q @ lv.k_route[i, r] * scale + lv.b_hat[i, r] == pytest.approx(exact, abs=1e-12)
            assert zo.node_scores(q, lv, np.array([i]), scale)[0] == pytest.approx(exact, abs=1e-12)


@pytest.mark.parametrize("level", [2, 3])
def test_parent_of_affine_children_equals_leaf_formula_over_span(level):
    """Keys constant over every level-(level-1) span: re-anchoring is exact, so the parent
    is the leaf formula over its span at its own rotated reference queries."""
    leaf, branch = 4, 4
    span_c = leaf * branch ** (level - 2)
    span_p = span_c * branch
    T = span_p * 5
    K = _keys(T, 10 + level, const_block=span_c)
    qref = _qref()
    tree = zo.build_tree(K, T, qref, depth=level, leaf=leaf, branch=branch, route_storage="f64",
                         state_storage="f64", inv_freq=FREQ)
    scale = 1 / math.sqrt(D)
    lv = tree.levels[level - 1]
    assert lv.n == 5
    for i in range(lv.n):
        q_p = zo.rope(qref, (i + 1) * span_p - 1, FREQ)
        k_hat, F, b_hat = zo.leaf_summary(K[i * span_p:(i + 1) * span_p], q_p, scale)
        np.testing.assert_allclose(lv.F[i], F, rtol=0, atol=1e-11)
        np.testing.assert_allclose(lv.k_state[i], k_hat, rtol=0, atol=1e-11)
        np.testing.assert_allclose(lv.b_hat[i], b_hat, rtol=0, atol=1e-10)
        # the same through the per-node merge with the children's rotated references
        child = tree.levels[level - 2]
        ids = np.arange(i * branch, (i + 1) * branch)
        q_c = zo.rope(qref[None], ((ids + 1) * span_c - 1)[:, None], FREQ)
        k2, F2, b2 = zo.merge_summaries(child.F[ids], child.k_state[ids], q_p, scale, q_child=q_c)
        np.testing.assert_allclose(F2, F, rtol=0, atol=1e-11)
        np.testing.assert_allclose(k2, k_hat, rtol=0, atol=1e-11)
        np.testing.assert_allclose(b2, b_hat, rtol=0, atol=1e-10)


def test_every_node_tangent_is_below_the_exact_log_mass():
    leaf, branch, depth = 4, 4, 3
    T = 64 * 3
    K = _keys(T, 20)
    qref = _qref()
    tree = zo.build_tree(K, T, qref, depth=depth, leaf=leaf, branch=branch, route_storage="f64",
                         state_storage="f64", inv_freq=FREQ)
    scale = 1 / math.sqrt(D)
    rng = np.random.default_rng(21)
    qs = [zo.rope(2 * rng.standard_normal(D), int(rng.integers(0, T)), FREQ) for _ in range(30)]
    for lvl in range(1, depth + 1):
        lv = tree.levels[lvl - 1]
        span = tree.span(lvl)
        for i in range(lv.n):
            anchors = [zo.rope(qref[r], (i + 1) * span - 1, FREQ) for r in range(qref.shape[0])]
            for q in qs + anchors:
                exact = zo.chunk_lse(q, K[i * span:(i + 1) * span], scale)
                assert zo.node_scores(q, lv, np.array([i]), scale)[0] <= exact + 1e-12
