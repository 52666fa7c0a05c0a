/*
 * zha.h - C ABI of the Zyphra Hierarchical Attention (ZHA) hot path on B200 (sm_100a).
 *
 * The method ("Subquadratic Attention with a Hierarchical Tree-Structured Indexer",
 * arXiv 2610.42112, and the ZHA summary page, Methodology) keeps the whole KV cache,
 * builds a tree of compressed key summaries over it, routes each query top-down with
 * adaptive top-p selection at every level, and attends exactly over the selected leaf
 * chunks plus the first key and the query's own partial chunk.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Ownership.  The caller allocates and frees every buffer.  The library never
 *    allocates, frees or synchronises; every call only enqueues kernels on `stream`
 *    (a cudaStream_t passed as void*; NULL is the legacy default stream).
 *  - Pointers.  Unless stated otherwise, every pointer argument is DEVICE memory of
 *    the current CUDA device.  `zha_geom*` and `zha_level_layout*` are host memory.
 *  - Layouts (row-major, innermost last):
 *      K, V      [B, Hkv, t_cap, d]  dtype  (a 64-key leaf chunk is one contiguous block)
 *      Q, O      [B, nq, Hq, d]      dtype
 *      q_pos     [B, nq]             int64  absolute position t of each query (its own key
 *                                           is already in the cache at position t)
 *      qref      [Hkv, R, d]         fp32   reference queries, shared by all nodes and levels;
 *                                           with g->rope_pairs = h > 0 followed by h fp32 rotary
 *                                           frequencies f_0..f_{h-1} (the model's RoPE table)
 *      leaf_ids  [B, nq, Hq, leaf_cap] int32 selected leaf-chunk ids, ascending
 *      leaf_cnt  [B, nq, Hq]         int32
 *      k_new, v_new [B, n_new, Hkv, d] dtype
 *    Query head h belongs to KV head h / (Hq / Hkv).
 *  - dtype.  ZHA_BF16 or ZHA_F32 for K, V, Q, O and the routing copy of the summaries.
 *    Softmax and accumulation run in fp32; tree summaries and routing scores in fp64.
 *  - Errors.  Problems visible on the host (bad geometry, null pointers, p outside (0,1],
 *    positions beyond t_cap, a workspace or tree buffer that is too small) return a
 *    non-zero zha_status before anything is enqueued.  A failed launch returns
 *    ZHA_ERR_CUDA.  Problems only visible on the device (leaf_cap overflow, an internal
 *    capacity exceeded) make the kernel write a non-zero zha_status into *dev_status
 *    (the first error wins; the library never clears it) and finish without touching
 *    memory out of bounds; the caller reads it after synchronising.  `dev_status` is a
 *    device int32 that the caller zeroes; it may not be NULL.
 *  - Determinism.  For fixed inputs every output is bit-identical from run to run: no
 *    floating-point atomics take part in any value.
 */
#ifndef ZHA_H
#define ZHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum zha_status {
  ZHA_OK = 0,
  ZHA_ERR_INVALID_ARG = 1,
  ZHA_ERR_UNSUPPORTED = 2,
  ZHA_ERR_CAPACITY = 3,
  ZHA_ERR_CUDA = 4,
  ZHA_ERR_DEVICE = 5
} zha_status;

typedef enum zha_dtype { ZHA_F32 = 0, ZHA_BF16 = 1 } zha_dtype;

/* Operation selector of zha_workspace_bytes. */
typedef enum zha_op {
  ZHA_OP_ROUTE = 1,   /* zha_route                                  */
  ZHA_OP_ATTN = 2,    /* zha_sparse_attn                            */
  ZHA_OP_DECODE = 3,  /* zha_decode (route + attention, nq = 1)     */
  ZHA_OP_DENSE = 4,   /* zha_dense_decode                           */
  ZHA_OP_FLAT = 5,    /* zha_flat_index (scores + select + attention) */
  ZHA_OP_PREFILL = 6  /* zha_prefill_attn (query tiles)             */
} zha_op;

/* Geometry of one attention layer and its tree (host struct).
 * d must be 128; leaf must be 64; 2 <= branch <= 64; 1 <= depth <= 8; R in {1, 2, 4, 8, 16};
 * 0 <= rope_pairs <= d / 2;
 * Hq % Hkv == 0 and Hq / Hkv <= 8; t_cap % leaf == 0; dtype a zha_dtype;
 * B * Hkv * t_cap * d * 4 <= 2^48 (bytes of the cache counted at 4 bytes per element),
 * else ZHA_ERR_UNSUPPORTED, so that no byte count the library forms can overflow. */
typedef struct zha_geom {
  int32_t B, Hq, Hkv, d;
  int32_t leaf;     /* keys per leaf chunk (level 1)                       */
  int32_t branch;   /* children per internal node                          */
  int32_t depth;    /* summary levels L; level l node spans leaf*branch^(l-1) */
  int32_t R;        /* reference queries per KV head                       */
  int64_t t_cap;    /* cache capacity per sequence, in tokens              */
  int32_t dtype;    /* zha_dtype                                           */
  int32_t rope_pairs; /* 0: no rotary positions; h in 1..d/2: reference queries are
                         rotated to each node's last position (see qref below)   */
} zha_geom;

/* A caller-owned device buffer. */
typedef struct zha_buf {
  void* base;
  size_t bytes;
} zha_buf;

/* Where one level of the tree lives inside the tree buffer (byte offsets from its base).
 * Node i of unit (b, h) at this level is entry ((b*Hkv + h)*n_cap + i) of each array. */
typedef struct zha_level_layout {
  int64_t n_cap;       /* node capacity per (b, h_kv): t_cap / span           */
  int64_t span;        /* keys per node                                        */
  size_t k_route_off;  /* [B, Hkv, n_cap, R, d] dtype: k_hat for routing       */
  size_t b_hat_off;    /* [B, Hkv, n_cap, R]    fp32: b_hat                     */
  size_t F_off;        /* [B, Hkv, n_cap, R]    fp32: merge state, log mass F   */
  size_t k_state_off;  /* [B, Hkv, n_cap, R, d] fp32: merge state, k_hat        */
} zha_level_layout;

/* Human-readable name of a status code (static string). */
const char* zha_status_str(int32_t status);

/* Validates a geometry; ZHA_OK or the reason it is rejected. */
zha_status zha_check_geom(const zha_geom* g);

/* Bytes of the tree buffer for this geometry (0 for an invalid geometry). */
size_t zha_tree_bytes(const zha_geom* g);

/* Layout of level `level` (1..depth) inside the tree buffer. */
zha_status zha_tree_level(const zha_geom* g, int32_t level, zha_level_layout* out);

/* Bytes of the workspace `op` needs for `nq` queries per sequence.  0 for an invalid
 * geometry, nq < 1, an unknown op, or B * nq * Hq * (t_cap / leaf + 2) * 8 > 2^48 (the
 * per-call arrays would not fit 64-bit byte counts); the entry points then return
 * ZHA_ERR_UNSUPPORTED (ZHA_ERR_INVALID_ARG for nq < 1) before anything is enqueued. */
size_t zha_workspace_bytes(const zha_geom* g, int32_t nq, int32_t op);

/* Leaf chunks a query can select at most (t_cap / leaf): a leaf_cap that never overflows. */
int64_t zha_leaf_cap(const zha_geom* g);

/*
 * zha_build_tree - summarise every full node over keys [0, T) of every (b, h_kv) unit.
 *
 * Leaves ("ZHA summary" page, Tree Construction; arXiv 2610.42112 §III-A): for each
 * 64-key chunk C and reference query q_hat_r,
 *   F_r = log sum_j exp(q_hat_r . k_j / sqrt(d)),   a_j = exp(q_hat_r . k_j / sqrt(d) - F_r),
 *   k_hat_r = sum_j a_j k_j,   b_hat_r = F_r - q_hat_r . k_hat_r / sqrt(d).
 * Parents (§III-B, App. D-B2, stable-state merge without re-anchoring): per reference,
 *   F_P = LSE_c F_c,  k_hat_P = sum_c exp(F_c - F_P) k_hat_c,  b_hat_P = F_P - q_hat . k_hat_P / sqrt(d).
 * Rotary positions (§III-B, models with RoPE), when g->rope_pairs = h > 0: the references
 * of a node are rotated to its last key position P (dims i and i + h, i < h, by the angle
 * P * f_i; dims >= 2h unrotated), and before a merge each child's log mass is moved to the
 * parent's rotated reference along its tangent plane, F_c += <k_hat_c, q_hat_P - q_hat_c> / sqrt(d).
 * The keys in the cache are taken as stored (already rotated by the model).
 * One launch for the leaves and one per parent level.  Arithmetic is fp64; the merge
 * state is stored as fp32, the routing k_hat in dtype, b_hat in fp32.
 *   K     [B, Hkv, t_cap, d] dtype; keys [0, T) are read.   0 <= T <= t_cap.
 *   qref  [Hkv, R, d] fp32 (+ g->rope_pairs fp32 frequencies).
 *   tree  at least zha_tree_bytes(g) bytes; nodes beyond T are left untouched.
 */
zha_status zha_build_tree(const zha_geom* g, const void* K, int64_t T, const float* qref,
                          zha_buf tree, int32_t* dev_status, void* stream);

/*
 * zha_append - write n_new tokens at positions [t_old, t_old + n_new) and summarise
 * every node that these tokens complete (arXiv 2610.42112 §III-A: a level-1 summary
 * every `leaf` tokens, a level-l one every leaf*branch^(l-1) tokens).
 *   k_new, v_new [B, n_new, Hkv, d] dtype (model layout), copied into K, V.
 *   Requires the tree to hold every full node over [0, t_old).  t_old + n_new <= t_cap.
 */
zha_status zha_append(const zha_geom* g, void* K, void* V, const void* k_new, const void* v_new,
                      int64_t t_old, int32_t n_new, const float* qref, zha_buf tree,
                      int32_t* dev_status, void* stream);

/*
 * zha_route - top-down adaptive top-p routing of every (query, query head)
 * ("ZHA summary" page, Routing; arXiv 2610.42112 §III-C, App. E-E).
 * For a query at position t a node is visible iff its span ends at or before
 * V(t) = leaf*floor(t/leaf).  The top level is the highest level with a visible node;
 * all its visible nodes are candidates.  At each level the node score is
 *   s(q) = max_r [ q . k_hat_r / sqrt(d) + b_hat_r ],
 * candidates are ordered by (score desc, node id asc) and the smallest prefix whose
 * softmax mass over the candidates reaches p is kept (all of them when p == 1).
 * The next level's candidates are the children of the kept nodes plus the visible
 * nodes whose parent is not visible.  The level-1 selection is S_1(q).
 *   Q          [B, nq, Hq, d] dtype;  q_pos [B, nq] int64, each < t_cap.
 *   p          in (0, 1].
 *   tree       built over at least [0, V(t)) for every query.
 *   leaf_ids   [B, nq, Hq, leaf_cap] ascending S_1(q); leaf_cnt [B, nq, Hq].
 *              More than leaf_cap leaves: the first leaf_cap are written, leaf_cnt =
 *              leaf_cap and *dev_status = ZHA_ERR_CAPACITY.
 *   level_cnt  nullable [B, nq, Hq, depth, 2] int32: (candidates, kept) at level l in
 *              slot l-1 (zeros above the query's top level).
 *   level_ids  nullable [B, nq, Hq, sum_{l>=2} n_cap(l)] int32: the kept nodes of level
 *              l >= 2, ascending, at offset sum_{2<=j<l} n_cap(j) (count in level_cnt).
 *   ws         at least zha_workspace_bytes(g, nq, ZHA_OP_ROUTE) bytes.
 */
zha_status zha_route(const zha_geom* g, const void* Q, const int64_t* q_pos, int32_t nq,
                     double p, zha_buf tree, int32_t* leaf_ids, int32_t* leaf_cnt,
                     int32_t leaf_cap, int32_t* level_cnt, int32_t* level_ids, zha_buf ws,
                     int32_t* dev_status, void* stream);

/*
 * zha_route_schedule - zha_route with one threshold per level.
 * Level l keeps the smallest prefix whose softmax mass reaches p_levels[l-1] instead of
 * a single p (arXiv 2610.42112 §VII, "Asymptotic length scaling": a constant p compounds
 * to p^L over L levels; a schedule such as p_l = p^(1/L) undoes that).  Candidates,
 * order, expansion and outputs are those of zha_route.
 *   p_levels  HOST array of g->depth doubles, each in (0, 1]; read before the call returns.
 *   Other arguments as zha_route.
 */
zha_status zha_route_schedule(const zha_geom* g, const void* Q, const int64_t* q_pos, int32_t nq,
                              const double* p_levels, zha_buf tree, int32_t* leaf_ids,
                              int32_t* leaf_cnt, int32_t leaf_cap, int32_t* level_cnt,
                              int32_t* level_ids, zha_buf ws, int32_t* dev_status, void* stream);

/*
 * zha_route_topk - the tree walk of zha_route with a fixed-count selector: level l keeps
 * its k_levels[l-1] best candidates in the same (score desc, node id asc) order, or all of
 * them when there are fewer (the fixed selection budget K of arXiv 2610.42112 App. D,
 * Table VI, which §III-C contrasts with top-p).  Candidates, expansion and outputs are
 * those of zha_route.
 *   k_levels  HOST array of g->depth int32 counts, each >= 1; read before the call returns.
 *   Other arguments as zha_route.
 */
zha_status zha_route_topk(const zha_geom* g, const void* Q, const int64_t* q_pos, int32_t nq,
                          const int32_t* k_levels, zha_buf tree, int32_t* leaf_ids, int32_t* leaf_cnt,
                          int32_t leaf_cap, int32_t* level_cnt, int32_t* level_ids, zha_buf ws,
                          int32_t* dev_status, void* stream);

/*
 * zha_sparse_attn - exact softmax attention over the index set
 * ("ZHA summary" page, Routing):  I(q) = {0} u (keys of the chunks in S_1(q)) u C_cur(q),
 * C_cur(q) = [V(t), t],   o(q) = sum_{j in I} softmax_j(q . k_j / sqrt(d)) v_j.
 * The G query heads of a KV head share one gather of the union of their chunks
 * (split-KV partials with d + 2 values each, then a log-sum-exp combine,
 * arXiv 2610.42112 App. D-B1).
 *   leaf_ids / leaf_cnt as produced by zha_route (ascending, each id < V(t)/leaf).
 *   O    [B, nq, Hq, d] dtype.   lse nullable [B, nq, Hq] fp32 (natural log).
 *   ws   at least zha_workspace_bytes(g, nq, ZHA_OP_ATTN) bytes.
 */
zha_status zha_sparse_attn(const zha_geom* g, const void* Q, const void* K, const void* V,
                           const int64_t* q_pos, int32_t nq, const int32_t* leaf_ids,
                           const int32_t* leaf_cnt, int32_t leaf_cap, void* O, float* lse,
                           zha_buf ws, int32_t* dev_status, void* stream);

/*
 * zha_prefill_attn - zha_sparse_attn for many queries per sequence (chunked prefill),
 * computed per query tile on the 5th-generation tensor cores.
 * Outputs are those of zha_sparse_attn: every query attends over its own index set
 * I(q) = {0} u (keys of the chunks in S_1(q)) u C_cur(q) ("ZHA summary" page, Routing).
 * arXiv 2610.42112, App. A-B (Table I) counts a tile of Q consecutive queries by the union
 * of the leaf lists of its Q queries x G heads; here a tile holds Qt = floor(128 / G)
 * consecutive queries of one sequence and the G heads of one KV head (Qt * G <= 128 rows
 * of one tcgen05 MMA), the tile's union is gathered once, and each row is masked to its
 * own chunks, the first key and its causal limit inside its own chunk.
 *   bf16 caches only (ZHA_ERR_UNSUPPORTED for fp32).
 *   Q, O [B, nq, Hq, d]; q_pos [B, nq] (required); leaf_ids / leaf_cnt as zha_route wrote them.
 *   lse  nullable [B, nq, Hq] fp32 (natural log).
 *   ws   at least zha_workspace_bytes(g, nq, ZHA_OP_PREFILL) bytes.
 * Softmax in fp32 (base 2, P rounded to bf16 for the second product), accumulation in fp32.
 */
zha_status zha_prefill_attn(const zha_geom* g, const void* Q, const void* K, const void* V,
                            const int64_t* q_pos, int32_t nq, const int32_t* leaf_ids,
                            const int32_t* leaf_cnt, int32_t leaf_cap, void* O, float* lse,
                            zha_buf ws, int32_t* dev_status, void* stream);

/*
 * zha_decode - one decode step for every sequence: append the new token at position T
 * (zha_append with n_new = 1), route its query (zha_route at t = T) and attend
 * (zha_sparse_attn).  T + 1 <= t_cap; the tree must hold every full node over [0, T).
 *   q     [B, 1, Hq, d];  k_new, v_new [B, 1, Hkv, d];  O [B, 1, Hq, d].
 *   leaf_ids / leaf_cnt receive S_1 as in zha_route.
 *   ws    at least zha_workspace_bytes(g, 1, ZHA_OP_DECODE) bytes.
 */
zha_status zha_decode(const zha_geom* g, const void* q, const void* k_new, const void* v_new,
                      void* K, void* V, int64_t T, const float* qref, double p, zha_buf tree,
                      int32_t* leaf_ids, int32_t* leaf_cnt, int32_t leaf_cap, void* O,
                      zha_buf ws, int32_t* dev_status, void* stream);

/*
 * zha_dense_decode - baseline: exact causal attention of each query over keys [0, t]
 * (flash-decode split-KV partials + combine, arXiv 2610.42112 App. D-A).
 *   Same layouts as zha_sparse_attn; ws >= zha_workspace_bytes(g, nq, ZHA_OP_DENSE).
 */
zha_status zha_dense_decode(const zha_geom* g, const void* Q, const void* K, const void* V,
                            const int64_t* q_pos, int32_t nq, void* O, float* lse, zha_buf ws,
                            int32_t* dev_status, void* stream);

/*
 * zha_flat_index - baseline: a flat indexer that scores every visible leaf chunk of
 * every query head by its exact log mass F_C(q) = log sum_{j in C} exp(q . k_j / sqrt(d))
 * ("ZHA summary" page, Tree Construction; reading every key, as the flat sparse-attention
 * indexers of arXiv 2610.42112 §I do), keeps the top-p chunks as zha_route does for one
 * level, and attends as zha_sparse_attn.  Scores are computed in fp32 (bf16 caches: on the
 * tensor cores, products of bf16 values accumulated in fp32), the log mass in fp64.
 *   ws >= zha_workspace_bytes(g, nq, ZHA_OP_FLAT).
 */
zha_status zha_flat_index(const zha_geom* g, const void* Q, const void* K, const void* V,
                          const int64_t* q_pos, int32_t nq, double p, int32_t* leaf_ids,
                          int32_t* leaf_cnt, int32_t leaf_cap, void* O, zha_buf ws,
                          int32_t* dev_status, void* stream);

/*
 * zha_sparse_attn_noalloc - zha_sparse_attn without a caller workspace.
 *
 * The paper has no counterpart: this entry point exists for callers that can pass the
 * library their inputs and outputs but cannot provide extra device memory (an engine's
 * plugin interface that hands over only the operator's buffers, or a process whose device
 * memory is wholly owned by another allocator).  The scratch lives in one file-scope
 * device array of ZHA_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU loading the library
 * holds until the process exits; the call allocates nothing.
 *   Arguments and result as zha_sparse_attn (same kernels; the split size is enlarged
 *   until the scratch fits, so values agree with zha_sparse_attn to fp32 rounding).
 *   Sizes whose scratch cannot fit even with the largest split return
 *   ZHA_ERR_CAPACITY before anything is enqueued.  At the largest split (1026 chunk ids per
 *   work item) a (sequence, query, KV head) unit needs about
 *     nr * (8216 + 528 G) + 528 G * ceil((t_cap/64 + 2) / 1026) bytes,
 *   nr = ceil((t_cap/64 + 1) / 1024), G = Hq / Hkv (the union lists of each block of 1024
 *   chunk ids, and one split partial of d + 4 floats per head and work item): with G = 8,
 *   366 units fit at t_cap = 128K, 255 at 240K and 60 at 1M; with G = 1, 614 at 128K.
 *   The first call on a device resolves the array's device address (cudaGetSymbolAddress
 *   with that device current); make that first call before any stream capture.  The
 *   address is kept per device index until the process exits: after cudaDeviceReset the
 *   library must be reloaded.
 *   Every call shares the array, and it keeps the previous call's contents (nothing in
 *   it needs to start at zero: every value read is written earlier in the same call).
 *   Calls that overlap on the GPU race on the array: issue them on one stream, or order
 *   them.
 */
#define ZHA_NOALLOC_SCRATCH_BYTES (16u << 20)
zha_status zha_sparse_attn_noalloc(const zha_geom* g, const void* Q, const void* K, const void* V,
                                   const int64_t* q_pos, int32_t nq, const int32_t* leaf_ids,
                                   const int32_t* leaf_cnt, int32_t leaf_cap, void* O, float* lse,
                                   int32_t* dev_status, void* stream);

/*
 * zha_check_bounded_wait - failure-detection check of the bounded device waits.
 * The paper has no counterpart: this call exercises the error path of the shared-memory
 * barrier waits that the TMA rings of the attention and flat-index kernels rely on.  It
 * launches one CTA whose first warp waits, with the rings' own bounded wait, on an
 * mbarrier that nothing ever completes and gives up after `polls` polls; it then sets
 * *dev_status = ZHA_ERR_DEVICE (the first error wins) and raises the CTA's abort flag,
 * as a ring kernel does.  A second warp waits on another never-completed barrier with a
 * 64 times larger limit and must stop early, on that flag.  The kernel ends normally:
 * no copy is in flight, nothing faults, and the context stays usable.
 *   polls       in [1, 2^32].
 *   out         device int64 [4]: the clock cycles each warp waited (warp 0, warp 1),
 *               then 1 / 0 for each warp: it returned without its barrier completing.
 *   dev_status  device int32 the caller zeroes.
 */
zha_status zha_check_bounded_wait(int64_t polls, int32_t* dev_status, int64_t* out, void* stream);

/* Number of kernels this library has enqueued since it was loaded (host counter). */
int64_t zha_launch_count(void);

/* The kernel and CUDA error behind the last ZHA_ERR_CUDA (static string, "no error"
 * before any failure; overwritten by the next failure). */
const char* zha_last_error(void);

/* Measurement hook.  Kernel ids for zha_trace. */
typedef enum zha_trace_kernel {
  ZHA_TRACE_ATTN = 1,        /* the split-KV gather kernel of the sparse / dense attention */
  ZHA_TRACE_ROUTE_SCORE = 2, /* the routing score kernel (every level launched on its own);
                                the flat indexer's chunk scores                             */
  ZHA_TRACE_ROUTE_SELECT = 3, /* the routing top-p select kernels (every level; both kinds) */
  ZHA_TRACE_ROUTE_FUSED = 4   /* the fused score + select of the small top levels of the tree
                                 (levels of at most 64 nodes per (b, h_kv)), one launch      */
} zha_trace_kernel;

/* Until n launches of kernel `which` have been traced, record start[i] just before and
 * stop[i] just after its i-th launch, on the stream of that launch.  start / stop are
 * host arrays of n cudaEvent_t (as void*) that stay valid until the launches are traced.
 * n = 0 switches tracing off.  Host-side only; not thread-safe against concurrent calls. */
void zha_trace(int32_t which, void* const* start, void* const* stop, int32_t n);

/* Launches of kernel `which` traced since the last zha_trace call. */
int32_t zha_trace_count(int32_t which);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H */
