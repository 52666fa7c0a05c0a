"""The oracle's pins catch planted mistakes.

Each case replaces one oracle function by a copy with one plausible slip (a dropped term, a
wrong sign, an index off by one, a transposed operand, an unnormalised weight, a wrong tie
order) and runs the pins of tests/test_oracle.py, tests/test_oracle_selectors.py or
tests/test_oracle_rope.py that cover it: at least one must fail.
The mistakes are planted in the oracle only, on the CPU.
"""
import numpy as np
import pytest

from oracle import zha_oracle as zo
from tests import test_oracle as pins
from tests import test_oracle_rope as rope_pins
from tests import test_oracle_selectors as sel_pins


def _golden():
    import json
    with open(pins.GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- planted mistakes


def leaf_bias_sign(Kc, qref, scale):
    k_hat, F, b_hat = _orig["leaf_summary"](Kc, qref, scale)
    return k_hat, F, F + np.sum(qref * k_hat, axis=-1) * scale


def leaf_uniform_weights(Kc, qref, scale):
    s = qref @ Kc.T * scale
    F = zo.lse(s, axis=-1)
    k_hat = np.tile(Kc.mean(0), (qref.shape[0], 1))
    return k_hat, F, F - np.sum(qref * k_hat, axis=-1) * scale


def leaf_no_scale_in_weights(Kc, qref, scale):
    s = qref @ Kc.T                                    # forgot the 1/sqrt(d)
    F = zo.lse(s * scale, axis=-1)
    a = np.exp(s - zo.lse(s, axis=-1)[:, None])
    k_hat = a @ Kc
    return k_hat, F, F - np.sum(qref * k_hat, axis=-1) * scale


def merge_unnormalised(F_c, k_hat_c, qref, scale):
    F = zo.lse(F_c, axis=0)
    w = np.exp(F_c)                                    # missing - F_P
    k_hat = np.einsum("cr,crd->rd", w, k_hat_c)
    return k_hat, F, F - np.sum(qref * k_hat, axis=-1) * scale


def merge_max_instead_of_lse(F_c, k_hat_c, qref, scale):
    F = np.max(F_c, axis=0)
    w = np.exp(F_c - zo.lse(F_c, axis=0)[None, :])
    k_hat = np.einsum("cr,crd->rd", w, k_hat_c)
    return k_hat, F, F - np.sum(qref * k_hat, axis=-1) * scale


def leaf_level_bias_sign(Kc, qn, scale):
    k_hat, F, b_hat = _orig["leaf_level"](Kc, qn, scale)
    return k_hat, F, F + np.sum(qn * k_hat, axis=-1) * scale


def leaf_level_unnormalised(Kc, qn, scale):
    s = np.matmul(np.broadcast_to(qn, (Kc.shape[0],) + qn.shape[1:]), np.swapaxes(Kc, 1, 2)) * scale
    F = zo.lse(s, axis=-1)
    k_hat = np.matmul(np.exp(s), Kc)                   # missing - F in the weights
    return k_hat, F, F - np.sum(qn * k_hat, axis=-1) * scale


def leaf_level_transposed(Kc, qn, scale):
    k_hat, F, b_hat = _orig["leaf_level"](Kc, qn, scale)
    return k_hat[:, ::-1], F, b_hat                    # references' k_hat swapped


def merge_level_bias_sign(F_c, k_hat_c, qP, scale):
    k_hat, F, b_hat = _orig["merge_level"](F_c, k_hat_c, qP, scale)
    return k_hat, F, F + np.sum(qP * k_hat, axis=-1) * scale


def merge_level_unnormalised(F_c, k_hat_c, qP, scale):
    F = zo.lse(F_c, axis=1)
    k_hat = np.einsum("ncr,ncrd->nrd", np.exp(F_c), k_hat_c)   # missing - F_P
    return k_hat, F, F - np.sum(qP * k_hat, axis=-1) * scale


def top_p_one_too_many(scores, ids, p):
    sel = _orig["top_p"](scores, ids, p)
    if sel.m < sel.n:
        order = np.lexsort((ids, -scores))
        return zo.Selection(np.sort(ids[order[:sel.m + 1]]), sel.m + 1, sel.n, sel.margin, sel.gap)
    return sel


def top_p_ties_descending(scores, ids, p):
    order = np.lexsort((-ids, -scores))                # wrong tie order
    s = scores[order]
    e = np.exp(s - s[0])
    cum = np.cumsum(e / e.sum())
    hit = np.nonzero(cum >= p)[0]
    m = len(ids) if p >= 1 or not len(hit) else int(hit[0]) + 1
    return zo.Selection(np.sort(ids[order[:m]]), m, len(ids), 0.0, 0.0)


def top_p_strict(scores, ids, p):
    order = np.lexsort((ids, -scores))
    s = scores[order]
    e = np.exp(s - s[0])
    cum = np.cumsum(e / e.sum())
    hit = np.nonzero(cum > p)[0]                       # > instead of >=
    m = len(ids) if p >= 1 or not len(hit) else int(hit[0]) + 1
    return zo.Selection(np.sort(ids[order[:m]]), m, len(ids), 0.0, 0.0)


def node_scores_sum_not_max(q, level, ids, scale):
    t = np.einsum("d,nrd->nr", q, level.k_route[ids]) * scale + level.b_hat[ids]
    return zo.lse(t, axis=-1)                          # a soft max instead of the max


def index_set_no_sink(leaves, t, leaf=64):
    v = leaf * (t // leaf)
    parts = [np.arange(v, t + 1, dtype=np.int64)]
    for c in leaves:
        parts.append(np.arange(c * leaf, (c + 1) * leaf, dtype=np.int64))
    return np.unique(np.concatenate(parts))


def index_set_partial_excludes_t(leaves, t, leaf=64):
    v = leaf * (t // leaf)
    parts = [np.array([0], np.int64), np.arange(v, t, dtype=np.int64)]
    for c in leaves:
        parts.append(np.arange(c * leaf, (c + 1) * leaf, dtype=np.int64))
    return np.unique(np.concatenate(parts))


def visible_count_off_by_one(t, span, leaf):
    return (leaf * (t // leaf) + leaf) // span         # counts the query's own chunk


def attention_no_scale(q, K, V, idx, block=1 << 20):
    Kx = zo._take_f64(K, np.asarray(idx))
    Vx = zo._take_f64(V, np.asarray(idx))
    z = Kx @ q
    e = np.exp(z - z.max())
    return (e @ Vx) / e.sum(), float(z.max() + np.log(e.sum()))


def round_bf16_via_f32(x):
    import torch
    return torch.from_numpy(np.asarray(x, np.float64).astype(np.float32)).to(torch.bfloat16).double().numpy()


def top_k_ties_descending(scores, ids, k):
    order = np.lexsort((-ids, -scores))                # wrong tie order
    m = min(int(k), len(ids))
    return zo.Selection(np.sort(ids[order[:m]]), m, len(ids), 0.0, 0.0)


def top_k_one_too_few(scores, ids, k):
    sel = _orig["top_k"](scores, ids, k)
    if sel.m > 1:
        order = np.lexsort((ids, -scores))
        return zo.Selection(np.sort(ids[order[:sel.m - 1]]), sel.m - 1, sel.n, sel.margin, sel.gap)
    return sel


def at_level_reversed(x, level):
    return x if np.ndim(x) == 0 else x[-level]         # level l read from the wrong end


def p_root_power_not_root(p, depth):
    return [float(p) ** depth] * depth


def reanchor_missing(F_c, k_hat_c, q_parent, q_child, scale):
    return F_c + 0.0 * np.sum(k_hat_c, axis=-1)        # the child's mass left at its own reference


def reanchor_sign(F_c, k_hat_c, q_parent, q_child, scale):
    return F_c + np.sum(k_hat_c * (q_child - q_parent), axis=-1) * scale


def node_anchor_first_key(i, span):
    return np.asarray(i, dtype=np.int64) * span         # rotated to the first key of the span


def rope_clockwise(x, pos, inv_freq):
    return _orig["rope"](x, -np.asarray(pos), inv_freq)  # the opposite sense of rotation


_orig = {"leaf_summary": zo.leaf_summary, "top_p": zo.top_p, "top_k": zo.top_k, "rope": zo.rope,
         "leaf_level": zo.leaf_level, "merge_level": zo.merge_level}


def _tree_pass_pins():
    for d in (8, 128):
        for rotary in (False, True):
            pins.test_build_tree_nodes_equal_the_per_node_formulas(d, rotary)


def _rope_tree_pins():
    rope_pins.test_leaf_tangent_exact_at_its_rotated_reference()
    for level in (2, 3):
        rope_pins.test_parent_of_affine_children_equals_leaf_formula_over_span(level)


def _route_pins():
    pins.test_expansion_with_orphans_hand_example()
    pins.test_p_one_routing_reproduces_dense_attention(8, 4096, 4095)
    pins.test_whole_route_levels_by_brute_force()


CASES = [
    ("leaf_summary", leaf_bias_sign,
     lambda: (pins.test_leaf_closed_form(_golden()), pins.test_leaf_bias_is_entropy_and_k_hat_is_gradient(8))),
    ("leaf_summary", leaf_uniform_weights,
     lambda: (pins.test_leaf_closed_form(_golden()), pins.test_leaf_bias_is_entropy_and_k_hat_is_gradient(8))),
    ("leaf_summary", leaf_no_scale_in_weights,
     lambda: pins.test_leaf_bias_is_entropy_and_k_hat_is_gradient(8)),
    ("merge_summaries", merge_unnormalised, lambda: pins.test_merge_closed_form(_golden())),
    ("merge_summaries", merge_max_instead_of_lse,
     lambda: (pins.test_merge_closed_form(_golden()), pins.test_merge_entropy_chain_rule())),
    ("leaf_level", leaf_level_bias_sign, _tree_pass_pins),
    ("leaf_level", leaf_level_unnormalised, _tree_pass_pins),
    ("leaf_level", leaf_level_transposed, _tree_pass_pins),
    ("merge_level", merge_level_bias_sign, _tree_pass_pins),
    ("merge_level", merge_level_unnormalised, _tree_pass_pins),
    ("top_p", top_p_one_too_many, lambda: [pins.test_top_p_is_minimal_by_brute_force(s) for s in range(25)]),
    ("top_p", top_p_ties_descending, lambda: pins.test_top_p_closed_form_with_ties(_golden(), "top_p_ties")),
    ("top_p", top_p_strict, lambda: pins.test_top_p_closed_form_with_ties(_golden(), "top_p_exact_boundary")),
    ("node_scores", node_scores_sum_not_max,
     lambda: pins.test_leaf_tangent_is_lower_bound_and_exact_at_reference(8)),
    ("index_set", index_set_no_sink, lambda: pins.test_index_set_closed_forms(_golden())),
    ("index_set", index_set_partial_excludes_t, lambda: pins.test_index_set_closed_forms(_golden())),
    ("visible_count", visible_count_off_by_one, _route_pins),
    ("attention", attention_no_scale, lambda: pins.test_p_one_routing_reproduces_dense_attention(8, 4096, 4095)),
    ("round_bf16", round_bf16_via_f32, pins.test_round_bf16_ties_to_even_and_no_double_rounding),
    ("top_k", top_k_ties_descending, lambda: [sel_pins.test_top_k_by_brute_force(s) for s in range(30)]),
    ("top_k", top_k_one_too_few, lambda: [sel_pins.test_top_k_by_brute_force(s) for s in range(30)]),
    ("_at_level", at_level_reversed,
     lambda: sel_pins.test_whole_route_with_per_level_parameters_by_brute_force("schedule")),
    ("p_root_schedule", p_root_power_not_root, sel_pins.test_p_root_schedule),
    ("reanchor", reanchor_missing, _rope_tree_pins),
    ("reanchor", reanchor_sign, _rope_tree_pins),
    ("node_anchor", node_anchor_first_key, _rope_tree_pins),
    ("rope", rope_clockwise, rope_pins.test_rope_is_complex_multiplication),
]


@pytest.mark.parametrize("name,mutant,check", CASES, ids=[f"{c[0]}:{c[1].__name__}" for c in CASES])
def test_pins_catch_planted_mistake(monkeypatch, name, mutant, check):
    monkeypatch.setattr(zo, name, mutant)
    with pytest.raises((AssertionError, ValueError)):
        check()


def test_unmutated_checks_pass():
    for _, _, check in CASES:
        check()
