"""CPU oracle of the Zyphra Hierarchical Attention (ZHA) hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or runs
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Plain numpy in float64, written step by step from the method's definitions:

* "ZHA summary" page (picx.dev), Methodology -> Tree Construction: chunk LSE
  F_C(q), tangent at a reference query (k_hat_r, b_hat_r), node score
  max_r t_r(q), recursive parents.
* "Subquadratic Attention with a Hierarchical Tree-Structured Indexer"
  (arXiv 2610.42112), §III-A (tree construction, b_hat is the entropy of the
  reference attention weights), §III-B (shared reference queries, estimated log
  attention mass of a child), §III-C (top-down top-p routing), App. D-B2
  (stable-state merge of the children's per-reference state, without
  Taylor/RoPE re-anchoring), App. E-E (nodes without complete parents join the
  frontier; the first key and the partial chunk are always read).
* Paper §III-B, models with RoPE: reference queries rotated to each node's
  last position; children re-anchored to the parent's rotated reference
  along their tangent planes before the merge (``rope``, ``reanchor``).
* "ZHA summary" page, Methodology -> Routing: m_l(q), the final index set
  I(q) = {0} u (union of selected leaf chunks) u C_cur(q), o(q) = Attn(q, K_I, V_I).

Readings taken where the pages are silent:
  * Tree nodes are stateless functions of the keys: a level-l node i spans
    keys [i*S_l, (i+1)*S_l), S_l = leaf * branch**(l-1); it exists once all its
    keys are in the cache.
  * A node is visible to a query at position t iff its span ends at or before
    V(t) = leaf * floor(t / leaf), the start of the query's own chunk.
  * Parents merge their children's per-reference state (LSE F and normalised
    k_hat) exactly; with no RoPE the re-anchoring term is zero, so in exact
    arithmetic the parent equals the leaf formula over its whole span.
  * Storage precision: the merge state (F, k_hat) is stored as fp32, the routing
    copy of k_hat in the KV dtype (bf16 or fp32), b_hat as fp32.  The oracle
    models these stores by rounding (round-to-nearest-even) exactly where they
    happen; ``storage="f64"`` switches the rounding off.
  * Top-p: candidates are ordered by (score desc, node index asc); m is the
    smallest prefix whose softmax mass reaches p, or all candidates if the
    rounded cumulative mass never does; p >= 1 keeps every candidate.
  * Scores, softmax and cumulative sums are float64 (the routing decision is
    made in float64 on both sides).
  * Selector variants (``route(..., p=schedule)`` and ``route(..., k=...)``):
    a per-level threshold p_l replaces the constant p level by level; the
    "p**(1/L)" schedule takes L = the configured depth; the fixed-count
    selector keeps the first min(K, n) candidates in the same (score desc,
    id asc) order.
  * Rotary variant (``build_tree(..., inv_freq=...)``): the pages name RoPE
    and partial RoPE but not the convention.  Dims (i, i + h), h =
    len(inv_freq), rotate by pos * inv_freq[i] and the remaining dims pass
    through (the "rotate half" pairing); the frequency table is an input (the
    model's), not computed here.  Keys arrive rotated; queries at their own
    position are rotated by the caller.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np

# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    Direct rounding of the float64 value to 8 significant bits (no detour via
    float32, which could round twice).  Values are finite; bf16 shares fp32's
    exponent range, and the subnormal range is treated like the normal range
    (never reached by the data here).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)               # x = m * 2**e, 0.5 <= |m| < 1
    r = np.rint(m * 256.0) / 256.0   # 8 significant bits, ties to even
    return np.ldexp(r, e)


def round_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(x: np.ndarray, storage: str) -> np.ndarray:
    if storage == "bf16":
        return round_bf16(x)
    if storage == "f32":
        return round_f32(x)
    if storage == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(storage)


# ---------------------------------------------------------------------------
# chunk log-mass and its tangent (summary page, Tree Construction; paper §III-A)
# ---------------------------------------------------------------------------


def lse(x: np.ndarray, axis=-1) -> np.ndarray:
    """log(sum(exp(x))) along ``axis``, shifted by the maximum."""
    m = np.max(x, axis=axis, keepdims=True)
    return np.squeeze(m, axis) + np.log(np.sum(np.exp(x - m), axis=axis))


def chunk_lse(q: np.ndarray, Kc: np.ndarray, scale: float) -> np.ndarray:
    """F_C(q) = log sum_j exp(q . k_j * scale).  q: [..., d], Kc: [C, d]."""
    return lse(q @ Kc.T * scale, axis=-1)


def leaf_summary(Kc: np.ndarray, qref: np.ndarray, scale: float):
    """Tangent-plane summary of one chunk for every reference query.

    k_hat_r = sum_j softmax_j(q_hat_r . k_j * scale) k_j
    F_r     = F_C(q_hat_r)
    b_hat_r = F_r - q_hat_r . k_hat_r * scale
    Kc: [C, d] keys, qref: [R, d].  Returns (k_hat [R, d], F [R], b_hat [R]).
    """
    s = qref @ Kc.T * scale                      # [R, C]
    F = lse(s, axis=-1)                          # [R]
    a = np.exp(s - F[:, None])                   # attention weights at q_hat_r
    k_hat = a @ Kc                               # [R, d]
    b_hat = F - np.sum(qref * k_hat, axis=-1) * scale
    return k_hat, F, b_hat


def rope(x: np.ndarray, pos, inv_freq) -> np.ndarray:
    """Rotary position embedding of ``x`` [..., d] at position(s) ``pos``.

    With h = len(inv_freq), dims i and i + h (i < h) are rotated together by the
    angle pos * inv_freq[i]:
      x'_i     = x_i cos - x_{i+h} sin,      x'_{i+h} = x_{i+h} cos + x_i sin;
    dims >= 2h pass through unchanged (partial rotary).  ``pos`` broadcasts
    against x.shape[:-1].  An empty ``inv_freq`` is the identity.
    """
    x = np.asarray(x, dtype=np.float64)
    f = np.asarray(inv_freq, dtype=np.float64)
    h = len(f)
    if h == 0:
        return x.copy()
    ang = np.asarray(pos, dtype=np.float64)[..., None] * f
    c, sn = np.cos(ang), np.sin(ang)
    out = np.array(np.broadcast_to(x, np.broadcast_shapes(x.shape, ang.shape[:-1] + x.shape[-1:])))
    x1, x2 = out[..., :h].copy(), out[..., h:2 * h].copy()
    out[..., :h] = x1 * c - x2 * sn
    out[..., h:2 * h] = x2 * c + x1 * sn
    return out


def node_anchor(i, span: int):
    """Position a node's reference queries are rotated to: the last key of its
    span [i * span, (i + 1) * span) (paper §III-B)."""
    return (np.asarray(i, dtype=np.int64) + 1) * span - 1


def reanchor(F_c: np.ndarray, k_hat_c: np.ndarray, q_parent: np.ndarray, q_child: np.ndarray,
             scale: float) -> np.ndarray:
    """A child's log mass F_c, estimated at its own reference query q_child, moved
    along its tangent plane to the parent's q_parent (paper §III-B): the
    compressed key's score at the parent's reference minus its score at the
    child's, F_c + <k_hat_c, q_parent - q_child> * scale.  Arrays broadcast;
    the last axis is d."""
    return F_c + np.sum(k_hat_c * (q_parent - q_child), axis=-1) * scale


def merge_summaries(F_c: np.ndarray, k_hat_c: np.ndarray, qref: np.ndarray, scale: float,
                    q_child: Optional[np.ndarray] = None):
    """Parent summary from its children's per-reference state.

    For each reference r independently (stable-state merge):
      F_P   = LSE_c F_c
      w_c   = exp(F_c - F_P)            (share of the parent's mass in child c)
      k_hat = sum_c w_c k_hat_c
      b_hat = F_P - q_hat_r . k_hat * scale
    F_c: [C, R], k_hat_c: [C, R, d].  Returns (k_hat [R, d], F [R], b_hat [R]).

    With rotary positions (paper §III-B) ``qref`` is the parent's rotated
    reference query q_hat_{r,P} and ``q_child`` [C, R, d] the children's
    q_hat_{r,c}: before the merge each child's log mass is moved to the parent's
    reference query along its tangent plane,
      F_c <- F_c + <k_hat_c, q_hat_{r,P} - q_hat_{r,c}> * scale.
    """
    if q_child is not None:
        F_c = reanchor(F_c, k_hat_c, qref[None, :, :], q_child, scale)
    F = lse(F_c, axis=0)                         # [R]
    w = np.exp(F_c - F[None, :])                 # [C, R]
    k_hat = np.einsum("cr,crd->rd", w, k_hat_c)
    b_hat = F - np.sum(qref * k_hat, axis=-1) * scale
    return k_hat, F, b_hat


# ---------------------------------------------------------------------------
# the tree of one (batch, KV head) unit
# ---------------------------------------------------------------------------


@dataclass
class Level:
    span: int                      # keys per node
    k_route: np.ndarray            # [n, R, d] routing copy of k_hat (stored precision)
    b_hat: np.ndarray              # [n, R]    (stored precision)
    F: np.ndarray                  # [n, R]    merge state (stored precision)
    k_state: np.ndarray            # [n, R, d] merge state (stored precision)

    @property
    def n(self) -> int:
        return self.k_route.shape[0]


@dataclass
class Tree:
    leaf: int
    branch: int
    depth: int
    levels: List[Level] = field(default_factory=list)   # levels[l-1] is level l

    def span(self, level: int) -> int:
        return self.leaf * self.branch ** (level - 1)


def _store_level(span, k_hat, F, b_hat, route_storage, state_storage):
    return Level(span=span,
                 k_route=round_to(k_hat, route_storage),
                 b_hat=round_to(b_hat, "f32" if state_storage != "f64" else "f64"),
                 F=round_to(F, state_storage),
                 k_state=round_to(k_hat, state_storage))


def rows_f64(K, a: int, b: int) -> np.ndarray:
    """Rows [a, b) of a key/value array as float64 (numpy or a CPU torch tensor)."""
    x = K[a:b]
    if hasattr(x, "double"):          # torch tensor: convert only this block
        return x.double().numpy()
    return np.asarray(x, dtype=np.float64)


def leaf_level(Kc: np.ndarray, qn: np.ndarray, scale: float):
    """``leaf_summary`` of n chunks at once, the formula unchanged.

    Kc: [n, C, d] keys of n chunks; qn: [n, R, d] the reference queries of each
    chunk (rotated per chunk) or [1, R, d] (one set for every chunk).
      s[n, r, c] = q_hat_{n,r} . k_{n,c} * scale,   F[n, r] = LSE_c s[n, r, c],
      a = exp(s - F),   k_hat[n, r] = sum_c a[n, r, c] k_{n,c},
      b_hat[n, r] = F[n, r] - q_hat_{n,r} . k_hat[n, r] * scale.
    Returns (k_hat [n, R, d], F [n, R], b_hat [n, R]).
    """
    if qn.shape[0] == 1:   # one q_hat for every chunk: a single matrix product, then a reshape
        n, C, d = Kc.shape
        s = np.swapaxes((Kc.reshape(-1, d) @ qn[0].T).reshape(n, C, -1), 1, 2) * scale
    else:
        s = np.matmul(qn, np.swapaxes(Kc, 1, 2)) * scale
    F = lse(s, axis=-1)
    a = np.exp(s - F[..., None])
    k_hat = np.matmul(a, Kc)                                # [n, r, d] = a[n, r, c] . K[n, c, d]
    b_hat = F - np.sum(qn * k_hat, axis=-1) * scale
    return k_hat, F, b_hat


def merge_level(F_c: np.ndarray, k_hat_c: np.ndarray, qP: np.ndarray, scale: float):
    """``merge_summaries`` of n parents at once, the formula unchanged.

    F_c: [n, C, R] and k_hat_c: [n, C, R, d], the (already re-anchored, with
    rotary positions) state of each parent's C children; qP: [n, R, d] the
    parents' reference queries or [1, R, d].
      F[n, r] = LSE_c F_c[n, c, r],   w = exp(F_c - F),
      k_hat[n, r] = sum_c w[n, c, r] k_hat_c[n, c, r],
      b_hat[n, r] = F[n, r] - q_hat_{n,r} . k_hat[n, r] * scale.
    Returns (k_hat [n, R, d], F [n, R], b_hat [n, R]).
    """
    F = lse(F_c, axis=1)                                     # [n, R]
    w = np.exp(F_c - F[:, None, :])                          # [n, C, R]
    k_hat = np.einsum("ncr,ncrd->nrd", w, k_hat_c)
    b_hat = F - np.sum(qP * k_hat, axis=-1) * scale
    return k_hat, F, b_hat


def build_tree(K, T: int, qref: np.ndarray, depth: int, leaf: int = 64,
               branch: int = 16, route_storage: str = "bf16", state_storage: str = "f32",
               block: int = 4096, inv_freq=None) -> Tree:
    """All full nodes over keys [0, T) of one unit.

    K: [>=T, d] keys (float64 values of the stored keys, or a CPU torch tensor
    read block by block), qref: [R, d].
    Level 1 summarises raw keys (``leaf_level``: ``leaf_summary`` per chunk);
    level l >= 2 merges the stored state of ``branch`` consecutive level-(l-1)
    nodes (``merge_level``: ``merge_summaries`` per parent).
    ``block`` only bounds the temporary memory of the vectorised leaf pass.

    ``inv_freq`` (rotary frequencies, see ``rope``; None or empty: no rotation)
    gives the RoPE variant of paper §III-B: node i of level l summarises at the
    reference queries rotated to its last position, q_hat_{r,i} =
    rope(q_hat_r, (i + 1) * span_l - 1), and a parent moves each child's log
    mass to its own rotated reference before the merge (``reanchor``).
    The keys are the cache's keys as stored (already rotated by the model).
    """
    rot = inv_freq is not None and len(inv_freq) > 0

    def rotated(level: int, n0: int, n1: int) -> np.ndarray:
        """q_hat of nodes [n0, n1) of ``level``: [n, R, d] (rotated) or [1, R, d]."""
        if not rot:
            return qref[None, :, :]
        last = node_anchor(np.arange(n0, n1, dtype=np.int64), tree.span(level))
        return rope(qref[None, :, :], last[:, None], inv_freq)

    d = K.shape[1]
    scale = 1.0 / math.sqrt(d)
    R = qref.shape[0]
    tree = Tree(leaf=leaf, branch=branch, depth=depth)
    n1 = T // leaf
    k1 = np.zeros((n1, R, d))
    F1 = np.zeros((n1, R))
    b1 = np.zeros((n1, R))
    for i0 in range(0, n1, block):
        i1 = min(n1, i0 + block)
        Kc = rows_f64(K, i0 * leaf, i1 * leaf).reshape(i1 - i0, leaf, d)
        k1[i0:i1], F1[i0:i1], b1[i0:i1] = leaf_level(Kc, rotated(1, i0, i1), scale)
    tree.levels.append(_store_level(leaf, k1, F1, b1, route_storage, state_storage))
    for lvl in range(2, depth + 1):
        child = tree.levels[-1]
        n = child.n // branch
        Fc = child.F[:n * branch].reshape(n, branch, R)
        kc = child.k_state[:n * branch].reshape(n, branch, R, d)
        qP = rotated(lvl, 0, n)                                 # [n or 1, R, d]
        if rot:                                                 # each child's log mass at the parent's q_hat
            qc = rotated(lvl - 1, 0, n * branch).reshape(n, branch, R, d)
            Fc = reanchor(Fc, kc, qP[:, None], qc, scale)
        kh, F, bh = merge_level(Fc, kc, qP, scale)
        tree.levels.append(_store_level(tree.span(lvl), kh, F, bh, route_storage, state_storage))
    return tree


# ---------------------------------------------------------------------------
# routing (summary page, Routing; paper §III-B normaliser over candidates, §III-C)
# ---------------------------------------------------------------------------


def node_scores(q: np.ndarray, level: Level, ids: np.ndarray, scale: float) -> np.ndarray:
    """s(q) = max_r [ q . k_hat_r * scale + b_hat_r ] for the nodes ``ids``."""
    t = np.einsum("d,nrd->nr", q, level.k_route[ids]) * scale + level.b_hat[ids]
    return np.max(t, axis=-1)


@dataclass
class Selection:
    ids: np.ndarray        # selected node ids, ascending
    m: int                 # number selected
    n: int                 # number of candidates
    margin: float          # min(cum_m - p, p - cum_{m-1}); inf when p >= 1 or m == n without reaching p
    gap: float             # pi_(m) - pi_(m+1) (inf if m == n)


def top_p(scores: np.ndarray, ids: np.ndarray, p: float) -> Selection:
    """Smallest prefix (scores desc, ids asc) whose softmax mass reaches p."""
    n = len(ids)
    if n == 0:
        return Selection(np.zeros(0, np.int64), 0, 0, math.inf, math.inf)
    order = np.lexsort((ids, -scores))
    s = scores[order]
    e = np.exp(s - s[0])
    pi = e / np.sum(e)
    cum = np.cumsum(pi)
    if p >= 1.0:
        m = n
        margin = math.inf
    else:
        hit = np.nonzero(cum >= p)[0]
        m = int(hit[0]) + 1 if len(hit) else n
        before = cum[m - 2] if m >= 2 else 0.0
        margin = min(cum[m - 1] - p, p - before) if len(hit) else abs(p - cum[-1])
    gap = pi[m - 1] - pi[m] if m < n else math.inf
    return Selection(np.sort(ids[order[:m]]), m, n, float(margin), float(gap))


def top_k(scores: np.ndarray, ids: np.ndarray, k: int) -> Selection:
    """The fixed-count selector: the first min(k, n) candidates in (score desc,
    id asc) order.

    The roofline-model variables of arXiv 2610.42112 (App. D, Table VI) name a
    fixed-count budget K beside the threshold p "when used by the chosen
    selector"; §III-C contrasts it with top-p.  ``margin`` is inf (no mass
    threshold); ``gap`` is pi_(m) - pi_(m+1) of the candidates' softmax, as for
    top-p, so that near-ties at the boundary are counted the same way.
    """
    n = len(ids)
    if n == 0 or k <= 0:
        return Selection(np.zeros(0, np.int64), 0, n, math.inf, math.inf)
    order = np.lexsort((ids, -scores))
    m = min(int(k), n)
    s = scores[order]
    e = np.exp(s - s[0])
    pi = e / np.sum(e)
    gap = pi[m - 1] - pi[m] if m < n else math.inf
    return Selection(np.sort(ids[order[:m]]), m, n, math.inf, float(gap))


def p_root_schedule(p: float, depth: int) -> List[float]:
    """Per-level thresholds p_l = p**(1/L), L = the configured depth, so that the
    product of the per-level thresholds over all L levels is p (arXiv
    2610.42112 §VII, "Asymptotic length scaling": a constant p gives a
    cumulative p**L; rescaling each level to p**(1/L) undoes it).  Index l-1
    holds level l."""
    return [float(p) ** (1.0 / depth)] * depth


def _at_level(x, level: int):
    """A per-level parameter: a scalar applies to every level; a sequence holds
    level l at index l-1."""
    return x if np.ndim(x) == 0 else x[level - 1]


def visible_count(t: int, span: int, leaf: int) -> int:
    """Full nodes of size ``span`` that end at or before the query's own chunk."""
    return (leaf * (t // leaf)) // span


@dataclass
class Route:
    top: int                                  # top level routed (0: nothing visible)
    cand: Dict[int, np.ndarray]               # level -> candidate ids (ascending)
    sel: Dict[int, Selection]                 # level -> selection
    leaves: np.ndarray                        # S_1(q), ascending chunk ids
    kept: Dict[int, np.ndarray] = field(default_factory=dict)   # level -> the ids expanded


def route(q: np.ndarray, t: int, tree: Tree, p, k=None, impose: Optional[Dict[int, np.ndarray]] = None) -> Route:
    """Top-down top-p routing of one query head at position ``t``.

    The top level is the highest level with a visible node; all its visible
    nodes are candidates.  Below it, the candidates are the children of the
    selected nodes plus the visible nodes whose parent is not visible.

    ``p`` is one threshold for every level (the pages' setting, §IV-A) or a
    per-level schedule (index l-1 = level l, e.g. ``p_root_schedule``).  With
    ``k`` (a count, or a per-level sequence of counts) each level keeps the
    k best candidates instead (``top_k``) and ``p`` is ignored.

    ``impose`` (for comparisons only: level -> ids) replaces the kept set of those
    levels by the given ids, which must be candidates of that level; the levels
    below are then routed from them.  ``sel[l]`` still holds the oracle's own
    selection of level l and ``kept[l]`` the set the expansion used.
    """
    d = q.shape[0]
    scale = 1.0 / math.sqrt(d)
    nvis = {l: visible_count(t, tree.span(l), tree.leaf) for l in range(1, tree.depth + 1)}
    for l in nvis:
        if l <= len(tree.levels) and nvis[l] > tree.levels[l - 1].n:
            raise ValueError(f"level {l}: {nvis[l]} nodes visible at t={t} but only "
                             f"{tree.levels[l - 1].n} built")
    top = max([l for l in nvis if nvis[l] >= 1], default=0)
    out = Route(top=top, cand={}, sel={}, leaves=np.zeros(0, np.int64))
    if top == 0:
        return out
    cand = np.arange(nvis[top], dtype=np.int64)
    for l in range(top, 0, -1):
        s = node_scores(q, tree.levels[l - 1], cand, scale)
        sel = top_p(s, cand, _at_level(p, l)) if k is None else top_k(s, cand, _at_level(k, l))
        out.cand[l] = cand
        out.sel[l] = sel
        kept = sel.ids
        if impose is not None and l in impose:
            kept = np.sort(np.asarray(impose[l], dtype=np.int64))
            if len(np.unique(kept)) != len(kept) or not np.all(np.isin(kept, cand)):
                raise ValueError(f"level {l}: imposed ids are not distinct candidates")
        out.kept[l] = kept
        if l > 1:
            children = (kept[:, None] * tree.branch + np.arange(tree.branch)[None, :]).ravel()
            orphans = np.arange(nvis[l] * tree.branch, nvis[l - 1], dtype=np.int64)
            cand = np.concatenate([children, orphans]).astype(np.int64)
    out.leaves = out.kept[1]
    return out


def index_set(leaves: Sequence[int], t: int, leaf: int = 64) -> np.ndarray:
    """I(q) = {0} u (keys of the selected leaf chunks) u C_cur(q), ascending.

    C_cur(q) holds the keys of the query's own chunk up to and including t.
    """
    v = leaf * (t // leaf)
    parts = [np.array([0], np.int64), np.arange(v, t + 1, dtype=np.int64)]
    for c in leaves:
        parts.append(np.arange(c * leaf, (c + 1) * leaf, dtype=np.int64))
    return np.unique(np.concatenate(parts))


# ---------------------------------------------------------------------------
# attention (summary page, Routing: o(q) = Attn(q, K_I, V_I))
# ---------------------------------------------------------------------------


def attention(q: np.ndarray, K, V, idx: np.ndarray, block: int = 1 << 20):
    """Softmax attention of q over the keys ``idx``.  Returns (o [d], lse).

    K, V: float64 arrays or CPU torch tensors.  The logits and the weighted sum
    of values are accumulated over ``block`` keys at a time only to bound the
    float64 temporaries of very long index sets.
    """
    scale = 1.0 / math.sqrt(q.shape[0])
    idx = np.asarray(idx)
    z = np.concatenate([_take_f64(K, idx[i:i + block]) @ q * scale for i in range(0, len(idx), block)])
    m = np.max(z)
    e = np.exp(z - m)
    o = np.zeros(q.shape[0])
    for i in range(0, len(idx), block):
        o += e[i:i + block] @ _take_f64(V, idx[i:i + block])
    return o / np.sum(e), float(m + np.log(np.sum(e)))


def _take_f64(X, idx: np.ndarray) -> np.ndarray:
    if hasattr(X, "double"):
        import torch
        return X[torch.from_numpy(np.ascontiguousarray(idx))].double().numpy()
    return np.asarray(X[idx], dtype=np.float64)


def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, t: int):
    """Causal dense attention over keys [0, t]."""
    return attention(q, K, V, np.arange(t + 1))


def flat_scores(q: np.ndarray, K: np.ndarray, t: int, leaf: int = 64) -> np.ndarray:
    """Exact chunk log-mass F_C(q) of every visible leaf chunk (flat indexer)."""
    d = q.shape[0]
    n = visible_count(t, leaf, leaf)
    if n == 0:
        return np.zeros(0)
    out = np.empty(n)
    step = 1 << 14
    for c0 in range(0, n, step):
        c1 = min(n, c0 + step)
        z = (rows_f64(K, c0 * leaf, c1 * leaf) @ q) / math.sqrt(d)
        out[c0:c1] = lse(z.reshape(c1 - c0, leaf), axis=-1)
    return out


def flat_select(q: np.ndarray, K: np.ndarray, t: int, p: float, leaf: int = 64) -> Selection:
    """Top-p over all visible leaf chunks scored by their exact log-mass."""
    s = flat_scores(q, K, t, leaf)
    return top_p(s, np.arange(len(s), dtype=np.int64), p)


# ---------------------------------------------------------------------------
# whole-path helpers over [B, Hkv, t, d] caches
# ---------------------------------------------------------------------------


def build_unit_trees(K: np.ndarray, T: int, qref: np.ndarray, depth: int,
                     route_storage: str, units: Optional[Sequence[tuple]] = None,
                     leaf: int = 64, branch: int = 16, state_storage: str = "f32"):
    """Trees of the (b, h_kv) ``units`` (all when None).  K: [B, Hkv, >=T, d]."""
    B, Hkv = K.shape[:2]
    units = units if units is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    return {u: build_tree(np.asarray(K[u[0], u[1]], np.float64), T, np.asarray(qref[u[1]], np.float64),
                          depth, leaf, branch, route_storage, state_storage) for u in units}


def decode_head(q: np.ndarray, K: np.ndarray, V: np.ndarray, t: int, tree: Tree, p: float):
    """Route one query head and attend over its index set.  Returns (route, o, lse)."""
    r = route(q, t, tree, p)
    o, l = attention(q, K, V, index_set(r.leaves, t, tree.leaf))
    return r, o, l
