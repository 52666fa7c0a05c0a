// Top-down adaptive top-p routing ("ZHA summary" page, Routing; arXiv 2610.42112 §III-C,
// App. E-E) and the flat exact-log-mass indexer used as a baseline.
//
// One level is two kernels over all (query, query head) pairs:
//   score : candidate ids of the level (top level: every visible node; below: the
//           children of the kept parents, then the visible nodes whose parent is not
//           visible) and their scores s = max_r [q . k_hat_r / sqrt(d) + b_hat_r], in fp64.
//   select: per query head, the smallest prefix of the candidates ordered by
//           (score desc, id asc) whose softmax mass reaches p.  Masses are fixed-point
//           integers 2^S * exp(s - max), so the sums are exact and order-free; the cutoff
//           is found by a radix select over the order-preserving 64-bit key of s, and
//           the kept ids are compacted in ascending order with a block scan.
#include <cooperative_groups.h>

#include "zha_internal.cuh"

namespace zha {

struct RouteGeom {
  int B, nq, Hq, Hkv, G, R, branch, depth;
  int64_t span[kMaxDepth + 2];   // span[l], l = 1..depth (span[depth+1] unused)
  int64_t ncap[kMaxDepth + 2];
  const int64_t* q_pos;          // [B, nq] or null
  int64_t pos_uniform;
  int64_t t_cap;
};

// Positions outside [0, t_cap) are rejected on the device: the query routes nothing.
__device__ __forceinline__ bool pos_ok(const RouteGeom& g, int64_t t) { return t >= 0 && t < g.t_cap; }

// Highest level with a visible node for a query at position t (0 if none).
__device__ __forceinline__ int top_level(const RouteGeom& g, int64_t t) {
  for (int l = g.depth; l >= 1; --l)
    if (visible_nodes(t, g.span[l]) >= 1) return l;
  return 0;
}

// ---------------------------------------------------------------------------
// score kernel: the G query heads of a (b, query, KV head) unit share every load.
// A work item is 128 candidate slots of one unit: at the unit's top level 128
// consecutive visible nodes; below it 128 / branch kept parents (their children) or the
// unit's orphans.  Each thread converts one node's summaries once and scores them for
// every head that has the node as a candidate; the score goes straight to that head's
// compact candidate list (children of its i-th kept parent at i*branch + c, orphans
// after all children), in ascending node order.
// ---------------------------------------------------------------------------

struct ScoreArgs {
  RouteGeom g;
  int level;
  const void* Q;                 // [B, nq, Hq, d]
  const void* k_route;           // level's routing k_hat [B, Hkv, ncap, R, d]
  const float* b_hat;            // [B, Hkv, ncap, R]
  const int* parents;            // kept ids of level+1, [nqh, C2]
  const int* parents_cnt;        // [nqh]
  int64_t C1, C2;
  int* cand_ids;                 // [nqh, C1]
  double* cand_score;            // [nqh, C1]
  int* cand_cnt;                 // [nqh]
  int64_t nblk;                  // work items per unit
  int32_t* dev_status;
};

constexpr int kScoreSlots = 128;                 // candidate slots per work item
#ifndef ZHA_SCORE_MIN_BLOCKS
#define ZHA_SCORE_MIN_BLOCKS 4                   // resident CTAs per SM the registers allow
#endif

// GPW = groups of 8 slots per warp: 4 (4 warps per item, for levels with many items) or 1
// (16 warps per item: a quarter of the dependent steps per warp, for the few items of the
// upper levels).
template <typename KT, int GPW>
__global__ void __launch_bounds__(kScoreSlots * 4 / GPW, GPW == 4 ? (sizeof(KT) == 2 ? ZHA_SCORE_MIN_BLOCKS : 3) : 1)
route_score_kernel(ScoreArgs a) {
  constexpr int kThreads = kScoreSlots * 4 / GPW;
  __shared__ __align__(16) double qfs[32][32];
  __shared__ int rank[kScoreSlots][kMaxG];       // per parent slot: rank in each head's list
  __shared__ int pcnt[kMaxG];
  __shared__ int n_kept;                         // kept parents of this item, over all heads
  const RouteGeom& g = a.g;
  const int tid = threadIdx.x;
  const int64_t units = (int64_t)g.B * g.nq * g.Hkv;
  const double scale = 1.0 / sqrt((double)kD);
  const int per_blk = kScoreSlots / g.branch;            // parents per work item
  for (int64_t w = blockIdx.x; w < units * a.nblk; w += gridDim.x) {
    const int64_t u = w % units;                         // block-major: the items of block 0
    const int64_t blk = w / units;                       // of every unit come first
    const int64_t bq = u / g.Hkv;
    const int hk = (int)(u % g.Hkv);
    const int64_t b = bq / g.nq;
    const int64_t qh0 = bq * g.Hq + (int64_t)hk * g.G;   // first head of the group
    const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
    if (!pos_ok(g, t)) {
      if (blk == 0 && tid == 0) set_status(a.dev_status, ZHA_ERR_INVALID_ARG);
      continue;
    }
    const int top = top_level(g, t);
    if (a.level > top) continue;                         // uniform over the CTA
    const int64_t nvis = visible_nodes(t, g.span[a.level]);
    const bool at_top = a.level == top;
    const int64_t npar = at_top ? 0 : visible_nodes(t, g.span[a.level + 1]);
    const int64_t orph_lo = npar * g.branch;
    const int64_t nb_par = (npar + per_blk - 1) / per_blk;
    // which slots this item covers
    int mode;                                            // 0 top nodes, 1 parents, 2 orphans
    if (at_top) {
      if (blk * kScoreSlots >= nvis) continue;
      mode = 0;
    } else if (blk < nb_par) {
      mode = 1;
    } else if (blk == nb_par && nvis > orph_lo) {
      mode = 2;
    } else if (blk == 0) {
      mode = 3;                                          // nothing to score; counts only
    } else {
      continue;
    }
    __syncthreads();                                     // smem reuse across items
    if (tid < g.G) pcnt[tid] = at_top ? 0 : a.parents_cnt[qh0 + tid];
    if (tid == 0) n_kept = 0;
    __syncthreads();
    if (blk == 0 && tid < g.G)
      a.cand_cnt[qh0 + tid] = (int)(at_top ? nvis : (int64_t)pcnt[tid] * g.branch + (nvis - orph_lo));
    if (mode == 3) continue;
    if (mode == 1) {
      // rank of each parent of this item in each head's kept list (-1: not kept): the kept
      // parents in [p0, p0 + per_blk) are consecutive entries of the head's ascending list,
      // from its lower bound of p0 on (one warp per head)
      const int64_t p0 = blk * per_blk;
      for (int i = tid; i < per_blk * g.G; i += kThreads) rank[i / g.G][i % g.G] = -1;
      __syncthreads();
      const int lane_ = tid & 31;
      for (int h = tid >> 5; h < g.G; h += kThreads / 32) {
        const int* lst = a.parents + (qh0 + h) * a.C2;
        const int cnt = pcnt[h];
        const int x = warp_lower_bound(lst, cnt, p0);
        int found = 0;
        for (int j = lane_; j < per_blk; j += 32) {
          if (x + j < cnt) {
            const int v = lst[x + j];
            if (v < p0 + per_blk && v < npar) {
              rank[v - p0][h] = x + j;
              ++found;
            }
          }
        }
        if (found) atomicAdd(&n_kept, found);
      }
      __syncthreads();
      // no head kept a parent of this item (sparse frontiers): nothing to score
      if (n_kept == 0) continue;
    }
    // B fragments of the mma: qfs[s][L] = q[head L/4][32 * (L%4) + s] (0 for heads >= G)
    for (int i = tid; i < 32 * 32; i += kThreads) {
      const int s2 = i / 32, L = i % 32, h = L >> 2;
      const KT* q = reinterpret_cast<const KT*>(a.Q) + qh0 * kD;
      qfs[s2][L] = h < g.G ? to_f64(q[h * kD + 32 * (L & 3) + s2]) : 0.0;
    }
    __syncthreads();
    // Scores on the fp64 tensor cores: each warp takes its 8*GPW slots as GPW groups of 8
    // nodes; D[8 nodes x 8 heads] += A[8 nodes x 4 dims] . B[4 dims x 8 heads] per
    // mma.m8n8k4.f64.  Lane L holds A[node L/4][dim 32*(L%4) + s] and B[dim][head L/4]
    // at k-step s (qf[s][L] in shared memory), so each lane reads 32 contiguous dims of
    // its node's row.  The (group, reference) steps are software-pipelined: the next
    // step's row is in flight while the current step's 32 mma run.
    const int lane = tid & 31, warp = tid >> 5;
    const int h0 = 2 * (lane & 3), h1 = h0 + 1;         // this lane's heads in D
    // node of this lane's row in group grp, and the heads that have it as a candidate
    auto slot_of = [&](int grp, int64_t& id, unsigned int& mask, int& j, int& c) {
      const int slot = (warp * GPW + grp) * 8 + (lane >> 2);
      mask = 0;
      j = 0;
      c = 0;
      if (mode == 0) {
        id = blk * kScoreSlots + slot;
        if (id < nvis) mask = (1u << g.G) - 1u;
      } else if (mode == 1) {
        j = slot / g.branch;
        c = slot % g.branch;
        id = (blk * per_blk + j) * g.branch + c;
        if (j < per_blk)
          for (int h = 0; h < g.G; ++h) mask |= (rank[j][h] >= 0 ? 1u : 0u) << h;
      } else {
        id = orph_lo + slot;
        if (id < nvis) mask = (1u << g.G) - 1u;
      }
    };
    // this warp's groups that hold a candidate of some head (warp-uniform); the steps run
    // over those groups only, so a sparse frontier costs fewer dependent steps
    uint32_t gsel = 0;                                   // 4 bits per selected group
    int ngrp = 0;
    for (int grp = 0; grp < GPW; ++grp) {
      int64_t id; unsigned int m; int jj, cc;
      slot_of(grp, id, m, jj, cc);
      if (__any_sync(0xffffffffu, m != 0)) gsel |= (uint32_t)grp << (4 * ngrp++);
    }
    if (ngrp == 0) continue;                             // warp-uniform
    constexpr int kVec = 16 / sizeof(KT);
    constexpr int kNv = 32 / kVec;                       // 16-byte vectors of 32 dims
    const int R = g.R;
    const int nsteps = ngrp * R;
    const int64_t node0 = (b * g.Hkv + hk) * g.ncap[a.level];
    // a step's row and its b_hat are loaded together, one step ahead of their use
    auto load_step = [&](uint4 (&v)[kNv], float& bh, int st) {
      const int gi = st / R, r = st - gi * R, grp = (int)((gsel >> (4 * gi)) & 15u);
      int64_t id; unsigned int m; int jj, cc;
      slot_of(grp, id, m, jj, cc);
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const KT*>(a.k_route) + ((node0 + id) * R + r) * kD + 32 * (lane & 3));
#pragma unroll
      for (int i = 0; i < kNv; ++i) v[i] = m ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      bh = m ? __ldg(a.b_hat + (node0 + id) * R + r) : 0.f;
    };
    double best0 = -INFINITY, best1 = -INFINITY;
    auto compute_step = [&](const uint4 (&v)[kNv], float bh, int st) {
      const int gi = st / R, r = st - gi * R, grp = (int)((gsel >> (4 * gi)) & 15u);
      double c0[4] = {0.0, 0.0, 0.0, 0.0}, c1[4] = {0.0, 0.0, 0.0, 0.0};   // 4 independent chains
#pragma unroll
      for (int s2 = 0; s2 < 32; ++s2) {
        const double av = (double)u4_elem<KT>(v[s2 / kVec], s2 % kVec);  // exact widening
        mma_f64(c0[s2 & 3], c1[s2 & 3], av, qfs[s2][lane]);
      }
      int64_t id; unsigned int m; int jj, cc;
      slot_of(grp, id, m, jj, cc);
      const double bb = (double)bh;
      best0 = fmax(best0, fma((c0[0] + c0[1]) + (c0[2] + c0[3]), scale, bb));
      best1 = fmax(best1, fma((c1[0] + c1[1]) + (c1[2] + c1[3]), scale, bb));
      if (r == R - 1) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int h = q ? h1 : h0;
          if (h < g.G && ((m >> h) & 1u)) {
            int64_t pos;
            if (mode == 0) pos = id;
            else if (mode == 1) pos = (int64_t)rank[jj][h] * g.branch + cc;
            else pos = (int64_t)pcnt[h] * g.branch + (id - orph_lo);
            double sc = q ? best1 : best0;
            if (sc == 0.0) sc = 0.0;                     // one zero (no -0.0) for the key order
            a.cand_ids[(qh0 + h) * a.C1 + pos] = (int)id;
            a.cand_score[(qh0 + h) * a.C1 + pos] = sc;
          }
        }
        best0 = best1 = -INFINITY;
      }
    };
    // three row buffers: the rows of the next two steps are in flight during each step
    uint4 vA[kNv], vB[kNv], vC[kNv];
    float bA, bB, bC;
    load_step(vA, bA, 0);
    if (nsteps > 1) load_step(vB, bB, 1);
    for (int st = 0; st < nsteps; st += 3) {
      if (st + 2 < nsteps) load_step(vC, bC, st + 2);
      compute_step(vA, bA, st);
      if (st + 3 < nsteps) load_step(vA, bA, st + 3);
      if (st + 1 < nsteps) compute_step(vB, bB, st + 1);
      if (st + 4 < nsteps) load_step(vB, bB, st + 4);
      if (st + 2 < nsteps) compute_step(vC, bC, st + 2);
    }
  }
}

// ---------------------------------------------------------------------------
// flat indexer scores: F_C(q) of every visible chunk, all G heads of a KV head per CTA
// ---------------------------------------------------------------------------

struct FlatArgs {
  RouteGeom g;
  const void* Q;
  const void* K;                 // [B, Hkv, t_cap, d]
  int64_t t_cap;
  int64_t C1;
  int* cand_ids;
  double* cand_score;
  int* cand_cnt;
  int64_t nblk;                  // chunk blocks (of 8 chunks) per unit
};

template <typename KT>
__global__ void __launch_bounds__(256) flat_score_kernel(FlatArgs a) {
  // 8 warps; warp w handles chunk (blk*8 + w) for every head of the unit
  __shared__ float qs[kMaxG][kD];
  const RouteGeom& g = a.g;
  const int64_t units = (int64_t)g.B * g.nq * g.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float scale = 1.0f / sqrtf((float)kD);
  for (int64_t w = blockIdx.x; w < units * a.nblk; w += gridDim.x) {
    const int64_t u = w / a.nblk, blk = w % a.nblk;
    const int64_t bq = u / g.Hkv;
    const int hk = (int)(u % g.Hkv);
    const int64_t b = bq / g.nq;
    const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
    const int64_t nvis = pos_ok(g, t) ? visible_nodes(t, kLeaf) : 0;
    if (blk == 0 && threadIdx.x < g.G) a.cand_cnt[bq * g.Hq + hk * g.G + threadIdx.x] = (int)nvis;
    if (blk * 8 >= nvis) continue;
    __syncthreads();
    for (int i = threadIdx.x; i < g.G * kD; i += blockDim.x) {
      const KT* q = reinterpret_cast<const KT*>(a.Q) + (bq * g.Hq + hk * g.G) * kD;
      qs[i / kD][i % kD] = to_f32(q[i]);
    }
    __syncthreads();
    const int64_t c = blk * 8 + warp;
    if (c >= nvis) continue;
    // lane handles keys lane and lane + 32 of the chunk
    const KT* k0 = reinterpret_cast<const KT*>(a.K) + ((b * g.Hkv + hk) * a.t_cap + c * kLeaf) * kD;
    float s0[kMaxG], s1[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) s0[h] = s1[h] = 0.f;
    const KT* ra = k0 + lane * kD;
    const KT* rb = k0 + (lane + 32) * kD;
    constexpr int kVec = 16 / sizeof(KT);
    for (int cc = 0; cc < kD; cc += kVec) {
      const uint4 va = *reinterpret_cast<const uint4*>(ra + cc);
      const uint4 vb = *reinterpret_cast<const uint4*>(rb + cc);
      const KT* ea = reinterpret_cast<const KT*>(&va);
      const KT* eb = reinterpret_cast<const KT*>(&vb);
#pragma unroll
      for (int uu = 0; uu < kVec; ++uu) {
        const float xa = to_f32(ea[uu]), xb = to_f32(eb[uu]);
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
          if (h < g.G) {
            s0[h] = fmaf(qs[h][cc + uu], xa, s0[h]);
            s1[h] = fmaf(qs[h][cc + uu], xb, s1[h]);
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h >= g.G) break;
      const float x0 = s0[h] * scale, x1 = s1[h] * scale;
      float m = fmaxf(x0, x1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float z = expf(x0 - m) + expf(x1 - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (lane == 0) {
        const int64_t qh = bq * g.Hq + hk * g.G + h;
        double F = (double)m + log((double)z);
        if (F == 0.0) F = 0.0;
        a.cand_ids[qh * a.C1 + c] = (int)c;
        a.cand_score[qh * a.C1 + c] = F;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// top-p select over one level's candidates with fixed-point masses; launch_select picks a
// warp, a CTA or a cluster of CTAs per query head from the level's frontier capacity
// ---------------------------------------------------------------------------

constexpr int kDigit = 11;
constexpr int kBuckets = 1 << kDigit;

struct SelectArgs {
  RouteGeom g;
  int level;
  int flat;                      // 1: a single level over all visible leaves
  double p;
  int64_t topk;                  // > 0: the fixed-count selector keeps the topk best; 0: top-p
  int mass_shift;                // fixed-point scale 2^mass_shift
  const int* cand_ids;
  const double* cand_score;
  unsigned long long* cand_mass;
  const int* cand_cnt;
  int64_t C1;
  int* out_ids;                  // [nqh, out_stride]
  int* out_cnt;                  // [nqh]
  int64_t out_stride;
  int out_cap;
  int* level_cnt;                // nullable [nqh, depth, 2]
  int* level_ids;                // nullable [nqh, level_ids_stride]
  int64_t level_ids_stride, level_ids_off, level_ids_cap;
  int32_t* dev_status;
};

__device__ __forceinline__ unsigned long long order_key(double s) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(s);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// ---------------------------------------------------------------------------
// The select of every level, in four steps per query head:
//   1. maximum M and minimum of the scores;
//   2. fixed-point masses E_i = round(2^S exp(s_i - M)), their exact total Z, and a
//      histogram of (count, mass) over linear buckets of [min, M] (the map from score to
//      bucket is monotone, so each bucket is an interval of the descending order);
//   3. the boundary bucket, where the cumulative mass from the top reaches ceil(p Z);
//      when it holds more than one candidate, an exact radix select on the 64-bit order
//      key of the score resolves it (digits below the common prefix of its keys);
//   4. ordered compaction of the kept candidates (ascending position = ascending id).
// The selected set is the one of the descending (score, then ascending id) order: the
// linear buckets only replace the first radix passes.
// ---------------------------------------------------------------------------

struct LinBuckets {
  double M, inv_w;
  int nb;
  __device__ __forceinline__ void init(double mx, double mn, int nbuckets) {
    M = mx;
    nb = nbuckets;
    const double r = mx - mn;
    const double iw = r > 0.0 ? (double)nbuckets / r : 0.0;
    inv_w = isfinite(iw) ? iw : 0.0;                 // 0: one bucket (the radix resolves it)
  }
  // nb - 1 for the highest scores, 0 for the lowest
  __device__ __forceinline__ int digit(double s) const {
    if (inv_w == 0.0) return nb - 1;
    const double x = (M - s) * inv_w;                // >= 0, monotone non-increasing in s
    return x < (double)(nb - 1) ? nb - 1 - (int)x : 0;
  }
};

// The cutoff, as every CTA / lane holds it after step 3.
struct Cutoff {
  bool keep_all;
  int d1;                        // boundary linear bucket
  int shift;                     // 64: every candidate of bucket d1 is kept
  unsigned long long pfx;        // key prefix (order_key >> shift) of the tie group
  unsigned long long need;       // candidates of the tie group kept, in position order
  unsigned int cnt_t;            // candidates of the tie group
};

// 0: dropped, 1: kept, 2: in the tie group
__device__ __forceinline__ int classify(const Cutoff& c, const LinBuckets& lb, double s) {
  if (c.keep_all) return 1;
  const int d = lb.digit(s);
  if (d != c.d1) return d > c.d1 ? 1 : 0;
  if (c.shift == 64) return 1;
  const unsigned long long kk = order_key(s) >> c.shift;
  return kk > c.pfx ? 1 : (kk == c.pfx ? 2 : 0);
}

__device__ __forceinline__ unsigned long long need_of(unsigned int cnt_b, unsigned long long mass_b,
                                                      unsigned long long tgt, unsigned long long above) {
  if (cnt_b <= 1) return 1;
  const unsigned long long e1 = mass_b / cnt_b;          // equal keys: equal masses
  unsigned long long need = e1 == 0 ? cnt_b : (tgt - above + e1 - 1) / e1;
  if (need < 1) need = 1;
  if (need > cnt_b) need = cnt_b;
  return need;
}

__device__ __forceinline__ unsigned long long target_of(double p, unsigned long long Z) {
  const double tg = ceil(p * (double)Z);
  unsigned long long tgt = tg < 1.0 ? 1ull : (unsigned long long)tg;
  return tgt > Z ? Z : tgt;
}

template <typename M>
__device__ __forceinline__ M lowest_bits(M m, long long r) {   // the r lowest set bits of m
  M out = 0;
  while (r > 0 && m) {
    const M b = m & (~m + 1);
    out |= b;
    m ^= b;
    --r;
  }
  return out;
}

// A boundary bucket of up to kMaxMembers candidates is resolved directly: its members
// (position, order key, mass) are gathered into a list and one warp walks them in the
// descending (key, then ascending position) order.  The member at which the cumulative
// mass from `above` first reaches tgt is the last kept; the cutoff becomes its key (pfx,
// shift 0), the members sharing that key (cnt_t) and how many of them, in position
// order, are kept (need).  Larger boundary buckets take the radix refinement.
constexpr int kMaxMembers = 32;

__device__ __forceinline__ void resolve_members(int m, const int* mpos, const unsigned long long* mkey,
                                                const unsigned long long* mmass, unsigned long long above,
                                                unsigned long long tgt, unsigned long long& pfx,
                                                unsigned long long& need, unsigned int& cnt_t) {
  const int lane = threadIdx.x & 31;
  const bool on = lane < m;
  const int p = on ? mpos[lane] : 0x7fffffff;
  const unsigned long long k = on ? mkey[lane] : 0ull;
  const unsigned long long e = on ? mmass[lane] : 0ull;
  unsigned long long cum = above;                      // mass up to and including this member
  for (int j = 0; j < m; ++j) {
    const unsigned long long kj = __shfl_sync(0xffffffffu, k, j);
    const int pj = __shfl_sync(0xffffffffu, p, j);
    const unsigned long long ej = __shfl_sync(0xffffffffu, e, j);
    if (kj > k || (kj == k && pj <= p)) cum += ej;
  }
  // the earliest member (in the order) whose cumulative mass reaches tgt
  const bool reach = on && cum >= tgt;
  unsigned long long kb = reach ? k : 0ull;
  bool any = reach;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long x = __shfl_xor_sync(0xffffffffu, kb, o);
    const bool ax = __shfl_xor_sync(0xffffffffu, any, o);
    if (ax && (!any || x > kb)) { kb = x; any = true; }
  }
  int pb = (reach && k == kb) ? p : 0x7fffffff;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pb = min(pb, __shfl_xor_sync(0xffffffffu, pb, o));
  pfx = kb;
  cnt_t = __popc(__ballot_sync(0xffffffffu, on && k == kb));
  need = __popc(__ballot_sync(0xffffffffu, on && k == kb && p <= pb));
}

// ---------------------------------------------------------------------------
// warp select: one warp per query head: 256 linear buckets, 8-bit radix digits, per-warp
// histograms in shared memory, warp shuffles for every reduction and scan.
// ---------------------------------------------------------------------------

constexpr int kWarpSelWarps = 4;
constexpr int kWDigit = 8;
constexpr int kWBuckets = 1 << kWDigit;
constexpr int kWarpCap = 1024;           // candidates a warp holds in shared memory

struct WarpSelSmem {                     // 4 warps: 62 KiB (dynamic shared memory)
  double sc[kWarpSelWarps][kWarpCap];
  int sid[kWarpSelWarps][kWarpCap];
  unsigned int cnt[kWarpSelWarps][kWBuckets];
  unsigned long long mass[kWarpSelWarps][kWBuckets];
  unsigned long long m_key[kWarpSelWarps][32], m_mass[kWarpSelWarps][32];
  int m_pos[kWarpSelWarps][32];
};

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned int warp_excl_scan(unsigned int v, unsigned int* total) {
  const int lane = threadIdx.x & 31;
  unsigned int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  *total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// The bucket where the cumulative mass from the top bucket, starting at `above`, reaches
// tgt.  Lane L owns the 8 buckets below kWBuckets - 8L.  Returns the bucket; `above`
// becomes the mass of the buckets above it.
__device__ __forceinline__ int warp_boundary(const unsigned long long* hmass, unsigned long long& above,
                                             unsigned long long tgt) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kWBuckets / 32;
  unsigned long long local = 0;
#pragma unroll
  for (int q = 0; q < kPer; ++q) local += hmass[kWBuckets - 1 - (lane * kPer + q)];
  unsigned long long x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const unsigned long long before = above + x - local;
  const bool mine = before < tgt && before + local >= tgt;
  int bstar = 0;
  unsigned long long above_new = 0;
  if (mine) {
    unsigned long long acc = before;
    for (int q = 0; q < kPer; ++q) {
      const int bkt = kWBuckets - 1 - (lane * kPer + q);
      if (acc + hmass[bkt] >= tgt) { bstar = bkt; above_new = acc; break; }
      acc += hmass[bkt];
    }
  }
  const unsigned int who = __ballot_sync(0xffffffffu, mine);
  const int src = who ? __ffs(who) - 1 : 0;
  above = __shfl_sync(0xffffffffu, above_new, src);
  return __shfl_sync(0xffffffffu, bstar, src);
}

__device__ __forceinline__ int* level_counts(const SelectArgs& a, int64_t qh) {
  return a.level_cnt ? a.level_cnt + (qh * a.g.depth + (a.level - 1)) * 2 : nullptr;
}

// Candidates of head qh at this level, or -1 when its query sees no node of the level
// (then `writer` records the empty selection).
__device__ __forceinline__ int head_candidates(const SelectArgs& a, int64_t qh, bool writer) {
  const RouteGeom& g = a.g;
  const int64_t t = query_pos(g.q_pos, g.pos_uniform, qh / g.Hq);
  const int top = !pos_ok(g, t) ? 0 : a.flat ? (visible_nodes(t, kLeaf) >= 1 ? 1 : 0) : top_level(g, t);
  if (a.level > top) {
    if (writer) {
      int* lc = level_counts(a, qh);
      if (lc) { lc[0] = 0; lc[1] = 0; }
      if (a.level == 1) a.out_cnt[qh] = 0;
    }
    return -1;
  }
  return a.cand_cnt[qh];
}

__device__ __forceinline__ unsigned long long mass_of(double s, double M, int shift) {
  return __double2ull_rn(ldexp(exp(s - M), shift));
}

// The selector's weights and target.  Top-p weighs a candidate by its fixed-point mass and
// targets ceil(p Z); the fixed-count selector (topk > 0) runs the same cutoff with a weight
// of 1 per candidate and the target topk, which keeps the topk first candidates in the same
// (score desc, id asc) order.
__device__ __forceinline__ unsigned long long sel_mass(const SelectArgs& a, double s, double M) {
  return a.topk > 0 ? 1ull : mass_of(s, M, a.mass_shift);
}
__device__ __forceinline__ bool sel_keeps_all(const SelectArgs& a, int64_t n) {
  return n == 0 || (a.topk > 0 ? a.topk >= n : a.p >= 1.0);
}
__device__ __forceinline__ unsigned long long sel_target(const SelectArgs& a, unsigned long long Z) {
  if (a.topk > 0) return (unsigned long long)a.topk < Z ? (unsigned long long)a.topk : Z;
  return target_of(a.p, Z);
}

// Writes the kept candidate `i` (id ids[i]) at output position pos.
__device__ __forceinline__ void emit_kept(const SelectArgs& a, int64_t qh, const int* ids, int i,
                                          unsigned int pos, bool& overflow) {
  const int id = ids[i];
  if ((int64_t)pos < a.out_cap) a.out_ids[qh * a.out_stride + pos] = id;
  else overflow = true;
  if (a.level_ids && a.level >= 2 && (int64_t)pos < a.level_ids_cap)
    a.level_ids[qh * a.level_ids_stride + a.level_ids_off + pos] = id;
}

// One warp per query head with its scores in shared memory (n <= kWarpCap): read once,
// every later pass walks shared memory; the compaction goes in rounds of 32 positions.
__global__ void __launch_bounds__(kWarpSelWarps * 32) route_select_warp_kernel(SelectArgs a) {
  extern __shared__ __align__(16) unsigned char wsel_raw[];
  WarpSelSmem& sm = *reinterpret_cast<WarpSelSmem*>(wsel_raw);
  const RouteGeom& g = a.g;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const unsigned int lt = (1u << lane) - 1u;
  double* sc = sm.sc[wid];
  int* sid = sm.sid[wid];
  unsigned int* hcnt = sm.cnt[wid];
  unsigned long long* hmass = sm.mass[wid];
  const int64_t nqh = (int64_t)g.B * g.nq * g.Hq;
  for (int64_t qh = (int64_t)blockIdx.x * kWarpSelWarps + wid; qh < nqh;
       qh += (int64_t)gridDim.x * kWarpSelWarps) {
    const int n = head_candidates(a, qh, lane == 0);
    if (n < 0) continue;
    if (n > kWarpCap) {                                  // the host picks a larger kernel
      if (lane == 0) set_status(a.dev_status, ZHA_ERR_CAPACITY);
      continue;
    }
    const double* s = a.cand_score + qh * a.C1;
    const int* ids = a.cand_ids + qh * a.C1;
    // 1. scores and ids into shared memory; maximum and minimum
    double mx = -INFINITY, mn = INFINITY;
#pragma unroll 4
    for (int i = lane; i < n; i += 32) {
      const double v = s[i];
      sc[i] = v;
      sid[i] = ids[i];
      mx = fmax(mx, v);
      mn = fmin(mn, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmax(mx, shfl_xor_f64(mx, o));
      mn = fmin(mn, shfl_xor_f64(mn, o));
    }
    // 2. masses, their total and the linear histogram
    LinBuckets lb;
    lb.init(mx, mn, kWBuckets);
#pragma unroll
    for (int q = 0; q < kWBuckets / 32; ++q) { hcnt[lane + 32 * q] = 0; hmass[lane + 32 * q] = 0; }
    __syncwarp();
    unsigned long long z = 0;
    for (int i = lane; i < n; i += 32) {
      const double v = sc[i];
      const unsigned long long e = sel_mass(a, v, mx);
      z += e;
      const int d = lb.digit(v);
      atomicAdd(&hcnt[d], 1u);
      atomicAdd(&hmass[d], e);
    }
    const unsigned long long Z = warp_sum_u64(z);
    __syncwarp();
    // 3. the cutoff
    Cutoff c{};
    c.keep_all = sel_keeps_all(a, n);
    c.shift = 64;
    if (!c.keep_all) {
      const unsigned long long tgt = sel_target(a, Z);
      unsigned long long above = 0;
      c.d1 = warp_boundary(hmass, above, tgt);
      unsigned int cnt_b = hcnt[c.d1];
      unsigned long long mass_b = hmass[c.d1];
      __syncwarp();
      if (cnt_b > 1 && cnt_b <= kMaxMembers) {
        // gather the boundary bucket's members and walk them in order
        unsigned int m = 0;
        for (int b0 = 0; b0 < n; b0 += 32) {
          const int i = b0 + lane;
          const bool mem = i < n && lb.digit(sc[i]) == c.d1;
          const unsigned int mb = __ballot_sync(0xffffffffu, mem);
          if (mem) {
            const unsigned int slot = m + __popc(mb & lt);
            sm.m_pos[wid][slot] = i;
            sm.m_key[wid][slot] = order_key(sc[i]);
            sm.m_mass[wid][slot] = sel_mass(a, sc[i], mx);
          }
          m += __popc(mb);
        }
        __syncwarp();
        c.shift = 0;
        resolve_members((int)m, sm.m_pos[wid], sm.m_key[wid], sm.m_mass[wid], above, tgt, c.pfx, c.need,
                        c.cnt_t);
        __syncwarp();
      } else if (cnt_b > 1) {
        // key range of the boundary bucket, then radix digits of the order key within it
        unsigned long long kmx = 0, kmn = ~0ull;
        for (int i = lane; i < n; i += 32) {
          const double v = sc[i];
          if (lb.digit(v) == c.d1) {
            const unsigned long long k = order_key(v);
            kmx = k > kmx ? k : kmx;
            kmn = k < kmn ? k : kmn;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long x = __shfl_xor_sync(0xffffffffu, kmx, o);
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, kmn, o);
          kmx = x > kmx ? x : kmx;
          kmn = y < kmn ? y : kmn;
        }
        if (kmx == kmn) {
          c.pfx = kmx;
          c.shift = 0;
        } else {
          int hi = 63 - __clzll((long long)(kmx ^ kmn));
          unsigned long long pfx = (hi == 63) ? 0ull : (kmx >> (hi + 1));
          while (true) {
            const int width = (hi + 1) < kWDigit ? (hi + 1) : kWDigit;
            const int lo = hi + 1 - width;
#pragma unroll
            for (int q = 0; q < kWBuckets / 32; ++q) { hcnt[lane + 32 * q] = 0; hmass[lane + 32 * q] = 0; }
            __syncwarp();
            for (int i = lane; i < n; i += 32) {
              const double v = sc[i];
              if (lb.digit(v) != c.d1) continue;
              const unsigned long long key = order_key(v);
              if ((hi == 63 ? 0ull : (key >> (hi + 1))) == pfx) {
                const unsigned int bkt = (unsigned int)((key >> lo) & ((1ull << width) - 1));
                atomicAdd(&hcnt[bkt], 1u);
                atomicAdd(&hmass[bkt], sel_mass(a, v, mx));
              }
            }
            __syncwarp();
            const int bstar = warp_boundary(hmass, above, tgt);
            cnt_b = hcnt[bstar];
            mass_b = hmass[bstar];
            pfx = (pfx << width) | (unsigned long long)bstar;
            __syncwarp();
            if (cnt_b <= 1 || lo == 0) { c.shift = lo; break; }
            hi = lo - 1;
          }
          c.pfx = pfx;
        }
        c.cnt_t = cnt_b;
        c.need = need_of(cnt_b, mass_b, tgt, above);
      }
    }
    // 4. ordered compaction, 32 positions per round
    const bool partial = c.shift != 64 && c.cnt_t > 1 && c.need < c.cnt_t;
    unsigned int written = 0, ties = 0;
    bool overflow = false;
    for (int b0 = 0; b0 < n; b0 += 32) {
      const int i = b0 + lane;
      const int k = i < n ? classify(c, lb, sc[i]) : 0;
      const unsigned int tb = __ballot_sync(0xffffffffu, k == 2);
      const bool keep = k == 1 || (k == 2 && (!partial || ties + __popc(tb & lt) < c.need));
      ties += __popc(tb);
      const unsigned int kb = __ballot_sync(0xffffffffu, keep);
      if (keep) emit_kept(a, qh, sid, i, written + __popc(kb & lt), overflow);
      written += __popc(kb);
    }
    if (overflow) set_status(a.dev_status, ZHA_ERR_CAPACITY);
    if (lane == 0) {
      a.out_cnt[qh] = (int64_t)written < a.out_cap ? (int)written : a.out_cap;
      int* lc = level_counts(a, qh);
      if (lc) { lc[0] = n; lc[1] = (int)written; }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// cluster select: one thread-block cluster (1..8 CTAs of T threads) per query head.  The
// cluster's rank-0 CTA sums the per-CTA maxima, totals and histograms through distributed
// shared memory and publishes every decision back into each CTA, so all CTAs take
// identical decisions.  Cluster barriers are hardware barriers (no spin loops).
// ---------------------------------------------------------------------------

constexpr int kClMaxCta = 8;

template <int T>
struct ClSmem {
  unsigned int cnt[kBuckets];
  unsigned long long mass[kBuckets];
  unsigned long long wsum[T / 32];
  unsigned long long wu[T / 32];
  double wd[T / 32];
  unsigned int wcnt[T / 32];
  unsigned int wdef[T / 32], wtie[T / 32], wkeep[T / 32];
  // per-CTA contributions, written into the rank-0 CTA by every rank
  unsigned long long slot_kmax[kClMaxCta], slot_kmin[kClMaxCta], slot_z[kClMaxCta];
  unsigned int slot_tie[kClMaxCta], slot_keep[kClMaxCta];
  // boundary-bucket members, gathered into rank 0
  unsigned int m_cnt;
  int m_pos[kMaxMembers];
  unsigned long long m_key[kMaxMembers], m_mass[kMaxMembers];
  // decisions published by rank 0
  unsigned long long d_above, d_mass_b, d_pfx, d_need;
  unsigned int d_cnt_b, d_cnt_t;
  int d_bstar;
};

// Barrier and shared-memory view of rank r: across the cluster (CL) or within the CTA.
template <bool CL>
__device__ __forceinline__ void csync() {
  if constexpr (CL) cooperative_groups::this_cluster().sync();
  else __syncthreads();
}
template <bool CL, typename S>
__device__ __forceinline__ S* peer(S& sm, int r) {
  if constexpr (CL) return cooperative_groups::this_cluster().map_shared_rank(&sm, r);
  else return &sm;
}

template <int T>
__device__ __forceinline__ double cl_block_max(double v, ClSmem<T>& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, shfl_xor_f64(v, o));
  __syncthreads();
  if (lane == 0) sm.wd[warp] = v;
  __syncthreads();
  double r = sm.wd[0];
  for (int i = 1; i < T / 32; ++i) r = fmax(r, sm.wd[i]);
  return r;
}

template <int T>
__device__ __forceinline__ unsigned long long cl_block_max_u64(unsigned long long v, ClSmem<T>& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long x = __shfl_xor_sync(0xffffffffu, v, o);
    v = x > v ? x : v;
  }
  __syncthreads();
  if (lane == 0) sm.wu[warp] = v;
  __syncthreads();
  unsigned long long r = sm.wu[0];
  for (int i = 1; i < T / 32; ++i) r = sm.wu[i] > r ? sm.wu[i] : r;
  return r;
}

template <int T>
__device__ __forceinline__ unsigned long long cl_block_sum(unsigned long long v, ClSmem<T>& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sm.wsum[warp] = v;
  __syncthreads();
  unsigned long long r = 0;
  for (int i = 0; i < T / 32; ++i) r += sm.wsum[i];
  return r;
}

// Cluster-wide boundary of the histograms every CTA has just filled: rank 0 sums them in
// rank order, finds the bucket where the cumulative mass from the top (starting at
// `above`) reaches tgt and publishes (bucket, mass above it, its count and mass) to every
// CTA.  Contains the two cluster barriers around the decision.
template <int T, bool CL>
__device__ __forceinline__ int cl_boundary(ClSmem<T>& sm, int CS, int cr, unsigned long long& above,
                                           unsigned long long tgt, unsigned int& cnt_b,
                                           unsigned long long& mass_b) {
  const int tid = threadIdx.x;
  csync<CL>();                                        // every CTA's histogram is complete
  if (cr == 0) {
    constexpr int kPer = kBuckets / T;
    unsigned long long bm[kPer];
    unsigned int bc[kPer];
    unsigned long long local = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int bkt = kBuckets - 1 - (tid * kPer + q);
      unsigned long long m2 = 0;
      unsigned int c2 = 0;
      for (int r = 0; r < CS; ++r) {
        ClSmem<T>* o = peer<CL>(sm, r);
        m2 += o->mass[bkt];
        c2 += o->cnt[bkt];
      }
      bm[q] = m2;
      bc[q] = c2;
      local += m2;
    }
    unsigned long long x = local;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sm.wsum[warp] = x;
    __syncthreads();
    unsigned long long before = above;
    for (int i = 0; i < warp; ++i) before += sm.wsum[i];
    before += x - local;
    if (before < tgt && before + local >= tgt) {
      unsigned long long acc = before;
      for (int q = 0; q < kPer; ++q) {
        if (acc + bm[q] >= tgt) {
          for (int r = 0; r < CS; ++r) {
            ClSmem<T>* o = peer<CL>(sm, r);
            o->d_bstar = kBuckets - 1 - (tid * kPer + q);
            o->d_above = acc;
            o->d_cnt_b = bc[q];
            o->d_mass_b = bm[q];
          }
          break;
        }
        acc += bm[q];
      }
    }
  }
  csync<CL>();                                           // decision published; histograms free
  above = sm.d_above;
  cnt_b = sm.d_cnt_b;
  mass_b = sm.d_mass_b;
  return sm.d_bstar;
}

template <int T>
__device__ __forceinline__ void cl_clear(ClSmem<T>& sm) {
  for (int i = threadIdx.x; i < kBuckets; i += T) { sm.cnt[i] = 0; sm.mass[i] = 0; }
  __syncthreads();
}

// Shared-memory-resident cluster select: CTA r of the cluster holds the contiguous slice
// [r*CAP, r*CAP + CAP) of the candidates' scores in (dynamic) shared memory, read once;
// every later pass walks shared memory.  The compaction gives warp w of each CTA a
// contiguous chunk of the slice, counted first, then written in rounds of 32 positions.
// n <= CS*CAP.
template <int T, int CAP, bool CL>
__global__ void __launch_bounds__(T) route_select_block_kernel(SelectArgs a) {
  constexpr bool CLK = CL;
  __shared__ ClSmem<T> sm;
  extern __shared__ __align__(16) double sc[];           // [CAP] scores, then [CAP] ids
  int CS = 1, cr = 0;
  if constexpr (CL) {
    CS = (int)cooperative_groups::this_cluster().num_blocks();
    cr = (int)cooperative_groups::this_cluster().block_rank();
  }
  ClSmem<T>* lead = peer<CL>(sm, 0);
  const RouteGeom& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  constexpr int W = T / 32;
  const unsigned int lt = (1u << lane) - 1u;
  const int64_t nqh = (int64_t)g.B * g.nq * g.Hq;
  const int64_t nclusters = gridDim.x / CS;
  int* sid = reinterpret_cast<int*>(sc + CAP);
  for (int64_t qh = blockIdx.x / CS; qh < nqh; qh += nclusters) {
    const int n = head_candidates(a, qh, cr == 0 && tid == 0);
    if (n < 0) continue;                                 // uniform over the cluster
    if (n > CS * CAP) {                                  // the host sizes the cluster from n_cap
      if (cr == 0 && tid == 0) set_status(a.dev_status, ZHA_ERR_CAPACITY);
      continue;
    }
    const int r0 = cr * CAP < n ? cr * CAP : n;
    const int len = (r0 + CAP < n ? r0 + CAP : n) - r0;
    const double* s = a.cand_score + qh * a.C1 + r0;
    const int* ids = a.cand_ids + qh * a.C1 + r0;

    // 1. scores into shared memory; maximum and minimum over the cluster
    double mx = -INFINITY, mn = INFINITY;
#pragma unroll 4
    for (int i = tid; i < len; i += T) {
      const double v = s[i];
      sc[i] = v;
      sid[i] = ids[i];
      mx = fmax(mx, v);
      mn = fmin(mn, v);
    }
    if (tid == 0) sm.m_cnt = 0;
    mx = cl_block_max(mx, sm);                           // (its barriers also publish sc)
    mn = -cl_block_max(-mn, sm);
    if (tid == 0) {
      lead->slot_kmax[cr] = order_key(mx);
      lead->slot_kmin[cr] = order_key(mn);
    }
    cl_clear(sm);
    csync<CL>();
    unsigned long long kmax = 0, kmin = ~0ull;
    for (int r = 0; r < CS; ++r) {
      const unsigned long long x = lead->slot_kmax[r], y = lead->slot_kmin[r];
      kmax = x > kmax ? x : kmax;
      kmin = y < kmin ? y : kmin;
    }
    const double M = __longlong_as_double((long long)((kmax >> 63) ? (kmax & 0x7fffffffffffffffull) : ~kmax));
    const double Mn = __longlong_as_double((long long)((kmin >> 63) ? (kmin & 0x7fffffffffffffffull) : ~kmin));

    // 2. masses, their total and the linear histogram
    LinBuckets lb;
    lb.init(M, Mn, kBuckets);
    unsigned long long z = 0;
    for (int i = tid; i < len; i += T) {
      const double v = sc[i];
      const unsigned long long e = sel_mass(a, v, M);
      z += e;
      const int d = lb.digit(v);
      atomicAdd(&sm.cnt[d], 1u);
      atomicAdd(&sm.mass[d], e);
    }
    z = cl_block_sum(z, sm);
    if (tid == 0) lead->slot_z[cr] = z;
    csync<CL>();
    unsigned long long Z = 0;
    for (int r = 0; r < CS; ++r) Z += lead->slot_z[r];

    // 3. the cutoff, with identical decisions in every CTA
    Cutoff c{};
    c.keep_all = sel_keeps_all(a, n);
    c.shift = 64;
    if (!c.keep_all) {
      const unsigned long long tgt = sel_target(a, Z);
      unsigned long long above = 0, mass_b = 0;
      unsigned int cnt_b = 0;
      c.d1 = cl_boundary<T, CLK>(sm, CS, cr, above, tgt, cnt_b, mass_b);
      if (cnt_b > 1 && cnt_b <= kMaxMembers) {
        // gather the boundary bucket's members into rank 0, which walks them in order
        for (int i = tid; i < len; i += T) {
          const double v = sc[i];
          if (lb.digit(v) == c.d1) {
            const unsigned int slot = atomicAdd(&lead->m_cnt, 1u);
            lead->m_pos[slot] = r0 + i;
            lead->m_key[slot] = order_key(v);
            lead->m_mass[slot] = sel_mass(a, v, M);
          }
        }
        csync<CL>();                                     // every member is in rank 0's list
        if (cr == 0 && wid == 0) {
          unsigned long long pfx, need;
          unsigned int cnt_t;
          resolve_members((int)sm.m_cnt, sm.m_pos, sm.m_key, sm.m_mass, above, tgt, pfx, need, cnt_t);
          if (lane < CS) {
            ClSmem<T>* o = peer<CL>(sm, lane);
            o->d_pfx = pfx;
            o->d_need = need;
            o->d_cnt_t = cnt_t;
          }
        }
        csync<CL>();                                     // decision published
        c.shift = 0;
        c.pfx = sm.d_pfx;
        c.need = sm.d_need;
        c.cnt_t = sm.d_cnt_t;
      } else if (cnt_b > 1) {
        unsigned long long kmx = 0, kmn = ~0ull;
        for (int i = tid; i < len; i += T) {
          const double v = sc[i];
          if (lb.digit(v) == c.d1) {
            const unsigned long long k = order_key(v);
            kmx = k > kmx ? k : kmx;
            kmn = k < kmn ? k : kmn;
          }
        }
        kmx = cl_block_max_u64(kmx, sm);
        kmn = ~cl_block_max_u64(~kmn, sm);
        if (tid == 0) { lead->slot_kmax[cr] = kmx; lead->slot_kmin[cr] = kmn; }
        cl_clear(sm);
        csync<CL>();
        kmx = 0;
        kmn = ~0ull;
        for (int r = 0; r < CS; ++r) {
          const unsigned long long x = lead->slot_kmax[r], y = lead->slot_kmin[r];
          kmx = x > kmx ? x : kmx;
          kmn = y < kmn ? y : kmn;
        }
        if (kmx == kmn) {
          c.pfx = kmx;
          c.shift = 0;
        } else {
          int hi = 63 - __clzll((long long)(kmx ^ kmn));
          unsigned long long pfx = (hi == 63) ? 0ull : (kmx >> (hi + 1));
          while (true) {
            const int width = (hi + 1) < kDigit ? (hi + 1) : kDigit;
            const int lo = hi + 1 - width;
            for (int i = tid; i < len; i += T) {
              const double v = sc[i];
              if (lb.digit(v) != c.d1) continue;
              const unsigned long long key = order_key(v);
              if ((hi == 63 ? 0ull : (key >> (hi + 1))) == pfx) {
                const unsigned int bkt = (unsigned int)((key >> lo) & ((1ull << width) - 1));
                atomicAdd(&sm.cnt[bkt], 1u);
                atomicAdd(&sm.mass[bkt], sel_mass(a, v, M));
              }
            }
            const int bstar = cl_boundary<T, CLK>(sm, CS, cr, above, tgt, cnt_b, mass_b);
            pfx = (pfx << width) | (unsigned long long)bstar;
            if (cnt_b <= 1 || lo == 0) { c.shift = lo; break; }
            cl_clear(sm);                                // rank 0 is done reading (cl_boundary)
            hi = lo - 1;
          }
          c.pfx = pfx;
        }
        c.cnt_t = cnt_b;
        c.need = need_of(cnt_b, mass_b, tgt, above);
      }
    }

    // 4. ordered compaction: warp w owns [c0, c1) of the slice (a multiple of 32 wide)
    const bool partial = c.shift != 64 && c.cnt_t > 1 && c.need < c.cnt_t;
    const int C = ((len + W - 1) / W + 31) & ~31;
    const int c0 = wid * C < len ? wid * C : len;
    const int c1 = c0 + C < len ? c0 + C : len;
    unsigned int ndef = 0, ntie = 0;
    for (int b0 = c0; b0 < c1; b0 += 32) {
      const int i = b0 + lane;
      const int k = i < c1 ? classify(c, lb, sc[i]) : 0;
      ndef += __popc(__ballot_sync(0xffffffffu, k == 1));
      ntie += __popc(__ballot_sync(0xffffffffu, k == 2));
    }
    if (lane == 0) { sm.wdef[wid] = ndef; sm.wtie[wid] = ntie; }
    __syncthreads();
    long long take = ntie;                               // ties this warp keeps
    if (partial) {
      unsigned int tie_before = 0, tie_cta = 0;
      for (int w2 = 0; w2 < W; ++w2) {
        if (w2 < wid) tie_before += sm.wtie[w2];
        tie_cta += sm.wtie[w2];
      }
      if (tid == 0) lead->slot_tie[cr] = tie_cta;
      csync<CL>();
      for (int r = 0; r < cr; ++r) tie_before += lead->slot_tie[r];
      take = (long long)c.need - (long long)tie_before;
      take = take < 0 ? 0 : (take > (long long)ntie ? (long long)ntie : take);
    }
    if (lane == 0) sm.wkeep[wid] = ndef + (unsigned int)take;
    __syncthreads();
    unsigned int pos = 0, keep_cta = 0;
    for (int w2 = 0; w2 < W; ++w2) {
      if (w2 < wid) pos += sm.wkeep[w2];
      keep_cta += sm.wkeep[w2];
    }
    if (tid == 0) lead->slot_keep[cr] = keep_cta;
    csync<CL>();
    unsigned int written = 0;
    for (int r = 0; r < CS; ++r) {
      const unsigned int k = lead->slot_keep[r];
      if (r < cr) pos += k;
      written += k;
    }
    bool overflow = false;
    unsigned int ties = 0;
    for (int b0 = c0; b0 < c1; b0 += 32) {
      const int i = b0 + lane;
      const int k = i < c1 ? classify(c, lb, sc[i]) : 0;
      const unsigned int tb = __ballot_sync(0xffffffffu, k == 2);
      const bool keep = k == 1 || (k == 2 && (long long)(ties + __popc(tb & lt)) < take);
      ties += __popc(tb);
      const unsigned int kb = __ballot_sync(0xffffffffu, keep);
      if (keep) emit_kept(a, qh, sid, i, pos + __popc(kb & lt), overflow);
      pos += __popc(kb);
    }
    if (overflow) set_status(a.dev_status, ZHA_ERR_CAPACITY);
    if (cr == 0 && tid == 0) {
      a.out_cnt[qh] = (int64_t)written < a.out_cap ? (int)written : a.out_cap;
      int* lc = level_counts(a, qh);
      if (lc) { lc[0] = n; lc[1] = (int)written; }
    }
    csync<CL>();                                      // slots, sc and smem reused by the next head
  }
}

// ---------------------------------------------------------------------------
// wide select: frontiers beyond the clusters' shared memory (more than 8 x 16896 candidates
// per head) as a chain of grid-wide kernels over (head, chunk of kWideChunk candidates), so
// that every SM works on a few heads' candidates; the heads' running state lives at the
// start of the head's row of the mass workspace (C1 x 8 bytes, C1 > 135168):
//   init -> maxima -> masses + linear histogram (per-CTA histograms added with global
//   atomics, integer sums: order-free) -> boundary bucket (a CTA per head) -> its members
//   gathered -> resolved (a CTA per head: the members sorted in shared memory, or, for a
//   boundary bucket of more than kWideMembers candidates, radix digits of the order key over
//   a stream of the head's candidates) -> keeps counted per chunk -> written in order.
// ---------------------------------------------------------------------------

constexpr int kWideChunk = 4096;
constexpr int kWideThreads = 256;                 // 16 candidates per thread
constexpr int kWideMembers = 4096;

enum : int { kWideSkip = -1, kWideDone = 0, kWideAll = 1, kWideGather = 2, kWideRadix = 3 };

struct WideHead {
  unsigned long long kmax, kmin, Z, tgt, above, mass_b, pfx, need;
  unsigned int mcount, cnt_b, cnt_t;
  int mode, d1, shift, n, pad;
  unsigned int cnt[kBuckets];
  unsigned long long mass[kBuckets];
  int m_pos[kWideMembers];
  unsigned long long m_key[kWideMembers], m_mass[kWideMembers];
  // followed by the chunks' keep counts: [nch] definite, then [nch] ties
};

__device__ __forceinline__ unsigned int* wide_chunks(const WideHead* h) {
  return reinterpret_cast<unsigned int*>(const_cast<WideHead*>(h) + 1);
}

__device__ __forceinline__ WideHead* wide_head(const SelectArgs& a, int64_t qh) {
  return reinterpret_cast<WideHead*>(a.cand_mass + qh * a.C1);
}

__device__ __forceinline__ double key_to_score(unsigned long long k) {
  return __longlong_as_double((long long)((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

__device__ __forceinline__ LinBuckets wide_buckets(const WideHead* h) {
  LinBuckets lb;
  lb.init(key_to_score(h->kmax), key_to_score(h->kmin), kBuckets);
  return lb;
}

__device__ __forceinline__ Cutoff wide_cutoff(const WideHead* h) {
  Cutoff c{};
  c.keep_all = h->mode == kWideAll;
  c.d1 = h->d1;
  c.shift = h->shift;
  c.pfx = h->pfx;
  c.need = h->need;
  c.cnt_t = h->cnt_t;
  return c;
}

// sum over the CTA (any T multiple of 32); the result is valid in every thread
template <typename V, int T>
__device__ __forceinline__ V wide_sum(V v, V* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  V r = 0;
  for (int w = 0; w < T / 32; ++w) r += scratch[w];
  return r;
}

__global__ void __launch_bounds__(kWideThreads) wide_init_kernel(SelectArgs a, int nch) {
  const int64_t qh = blockIdx.x;
  WideHead* h = wide_head(a, qh);
  const int n = head_candidates(a, qh, threadIdx.x == 0);
  if (threadIdx.x == 0) {
    h->n = n;
    h->mode = n < 0 ? kWideSkip : kWideDone;
    h->kmax = 0ull;
    h->kmin = ~0ull;
    h->Z = 0ull;
    h->mcount = 0u;
    h->shift = 64;
  }
  if (n < 0) return;
  for (int i = threadIdx.x; i < kBuckets; i += kWideThreads) { h->cnt[i] = 0u; h->mass[i] = 0ull; }
  for (int i = threadIdx.x; i < 2 * nch; i += kWideThreads) wide_chunks(h)[i] = 0u;
}

__global__ void __launch_bounds__(kWideThreads) wide_minmax_kernel(SelectArgs a, int nch) {
  __shared__ unsigned long long red[kWideThreads / 32];
  const int64_t qh = blockIdx.x / nch;
  const int c = (int)(blockIdx.x % nch);
  const WideHead* h = wide_head(a, qh);
  if (h->mode == kWideSkip) return;
  const int i0 = c * kWideChunk;
  const int i1 = min(h->n, i0 + kWideChunk);
  if (i0 >= i1) return;
  const double* s = a.cand_score + qh * a.C1;
  unsigned long long kx = 0ull, kn = ~0ull;
#pragma unroll 8
  for (int i = i0 + threadIdx.x; i < i1; i += kWideThreads) {
    const unsigned long long k = order_key(s[i]);
    kx = k > kx ? k : kx;
    kn = k < kn ? k : kn;
  }
  // maxima of the keys (the minimum as the complement's maximum)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long x = __shfl_xor_sync(0xffffffffu, kx, o), y = __shfl_xor_sync(0xffffffffu, kn, o);
    kx = x > kx ? x : kx;
    kn = y < kn ? y : kn;
  }
  if (lane == 0) red[warp] = kx;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kWideThreads / 32; ++w) kx = red[w] > kx ? red[w] : kx;
    atomicMax(&wide_head(a, qh)->kmax, kx);
  }
  __syncthreads();
  if (lane == 0) red[warp] = kn;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kWideThreads / 32; ++w) kn = red[w] < kn ? red[w] : kn;
    atomicMin(&wide_head(a, qh)->kmin, kn);
  }
}

__global__ void __launch_bounds__(kWideThreads) wide_hist_kernel(SelectArgs a, int nch) {
  __shared__ unsigned int cnt[kBuckets];
  __shared__ unsigned long long mass[kBuckets];
  __shared__ unsigned long long red[kWideThreads / 32];
  const int64_t qh = blockIdx.x / nch;
  const int c = (int)(blockIdx.x % nch);
  WideHead* h = wide_head(a, qh);
  if (h->mode == kWideSkip) return;
  const int i0 = c * kWideChunk;
  const int i1 = min(h->n, i0 + kWideChunk);
  if (i0 >= i1) return;
  const LinBuckets lb = wide_buckets(h);
  const double M = lb.M;
  for (int i = threadIdx.x; i < kBuckets; i += kWideThreads) { cnt[i] = 0u; mass[i] = 0ull; }
  __syncthreads();
  const double* s = a.cand_score + qh * a.C1;
  unsigned long long z = 0ull;
#pragma unroll 4
  for (int i = i0 + threadIdx.x; i < i1; i += kWideThreads) {
    const double v = s[i];
    const unsigned long long e = sel_mass(a, v, M);
    z += e;
    const int d = lb.digit(v);
    atomicAdd(&cnt[d], 1u);
    atomicAdd(&mass[d], e);
  }
  z = wide_sum<unsigned long long, kWideThreads>(z, red);    // contains the barriers
  if (threadIdx.x == 0) atomicAdd(&h->Z, z);
  for (int i = threadIdx.x; i < kBuckets; i += kWideThreads) {
    if (cnt[i]) {
      atomicAdd(&h->cnt[i], cnt[i]);
      atomicAdd(&h->mass[i], mass[i]);
    }
  }
}

// One CTA of 1024 threads per head: the boundary bucket of the global histogram.
__global__ void __launch_bounds__(1024) wide_boundary_kernel(SelectArgs a) {
  __shared__ ClSmem<1024> sm;
  const int64_t qh = blockIdx.x;
  WideHead* h = wide_head(a, qh);
  if (h->mode == kWideSkip) return;
  if (sel_keeps_all(a, h->n)) {
    if (threadIdx.x == 0) h->mode = kWideAll;
    return;
  }
  for (int i = threadIdx.x; i < kBuckets; i += 1024) { sm.cnt[i] = h->cnt[i]; sm.mass[i] = h->mass[i]; }
  const unsigned long long tgt = sel_target(a, h->Z);
  unsigned long long above = 0ull, mass_b = 0ull;
  unsigned int cnt_b = 0u;
  const int d1 = cl_boundary<1024, false>(sm, 1, 0, above, tgt, cnt_b, mass_b);   // syncs first
  if (threadIdx.x == 0) {
    h->tgt = tgt;
    h->d1 = d1;
    h->above = above;
    h->cnt_b = cnt_b;
    h->mass_b = mass_b;
    h->shift = 64;                               // a single candidate: the whole bucket is kept
    h->mode = cnt_b <= 1 ? kWideDone : (cnt_b <= (unsigned)kWideMembers ? kWideGather : kWideRadix);
  }
}

__global__ void __launch_bounds__(kWideThreads) wide_gather_kernel(SelectArgs a, int nch) {
  const int64_t qh = blockIdx.x / nch;
  const int c = (int)(blockIdx.x % nch);
  WideHead* h = wide_head(a, qh);
  if (h->mode != kWideGather) return;
  const int i0 = c * kWideChunk;
  const int i1 = min(h->n, i0 + kWideChunk);
  const LinBuckets lb = wide_buckets(h);
  const int d1 = h->d1;
  const double* s = a.cand_score + qh * a.C1;
  for (int i = i0 + threadIdx.x; i < i1; i += kWideThreads) {
    const double v = s[i];
    if (lb.digit(v) != d1) continue;
    const unsigned int slot = atomicAdd(&h->mcount, 1u);   // < cnt_b <= kWideMembers
    if (slot >= (unsigned)kWideMembers) continue;          // (the histogram counted them all)
    h->m_pos[slot] = i;
    h->m_key[slot] = order_key(v);
    h->m_mass[slot] = sel_mass(a, v, lb.M);
  }
}

// One CTA of 1024 threads per head: the boundary bucket resolved.
__global__ void __launch_bounds__(1024) wide_resolve_kernel(SelectArgs a) {
  extern __shared__ __align__(16) unsigned char wide_raw[];
  __shared__ ClSmem<1024> sm;
  const int64_t qh = blockIdx.x;
  WideHead* h = wide_head(a, qh);
  const int tid = threadIdx.x;
  const int mode = h->mode;
  if (mode != kWideGather && mode != kWideRadix) return;
  const unsigned long long tgt = h->tgt;
  unsigned long long above = h->above;
  if (mode == kWideGather) {
    // sort the members by (key descending, position ascending), then walk their masses
    unsigned long long* key = reinterpret_cast<unsigned long long*>(wide_raw);
    unsigned long long* ms = key + kWideMembers;
    int* pos = reinterpret_cast<int*>(ms + kWideMembers);
    const int m = (int)(h->mcount < (unsigned)kWideMembers ? h->mcount : (unsigned)kWideMembers);
    int P = 1;
    while (P < m) P <<= 1;
    for (int i = tid; i < P; i += 1024) {
      const bool on = i < m;
      key[i] = on ? h->m_key[i] : 0ull;            // 0 is below every order key of a score
      pos[i] = on ? h->m_pos[i] : 0x7fffffff;
      ms[i] = on ? h->m_mass[i] : 0ull;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < P; i += 1024) {
          const int l = i ^ j;
          if (l > i) {
            const bool first_before = key[i] > key[l] || (key[i] == key[l] && pos[i] < pos[l]);
            const bool up = (i & k) == 0;          // this pair's run is in (descending) order
            if (first_before != up) {
              const unsigned long long tk = key[i]; key[i] = key[l]; key[l] = tk;
              const int tp = pos[i]; pos[i] = pos[l]; pos[l] = tp;
              const unsigned long long tm = ms[i]; ms[i] = ms[l]; ms[l] = tm;
            }
          }
        }
        __syncthreads();
      }
    }
    // the first member (in order) whose cumulative mass from `above` reaches tgt: a block
    // scan of the sorted masses, thread t owning the consecutive members [4t, 4t + 4)
    __shared__ int s_cidx;
    __shared__ unsigned int s_cnt, s_need;
    constexpr int kPerT = kWideMembers / 1024;
    unsigned long long loc[kPerT], lsum = 0;
#pragma unroll
    for (int q = 0; q < kPerT; ++q) {
      const int i = tid * kPerT + q;
      loc[q] = i < m ? ms[i] : 0ull;
      lsum += loc[q];
    }
    if (tid == 0) { s_cidx = m - 1; s_cnt = 0u; s_need = 0u; }
    unsigned long long x = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
      if ((tid & 31) >= o) x += y;
    }
    if ((tid & 31) == 31) sm.wsum[tid >> 5] = x;
    __syncthreads();
    unsigned long long acc = above + x - lsum;
    for (int w = 0; w < (tid >> 5); ++w) acc += sm.wsum[w];
#pragma unroll
    for (int q = 0; q < kPerT; ++q) {
      const int i = tid * kPerT + q;
      acc += loc[q];
      if (i < m && acc >= tgt) { atomicMin(&s_cidx, i); break; }
    }
    __syncthreads();
    const unsigned long long kc = key[s_cidx];
    const int pc = pos[s_cidx];
    unsigned int ct = 0, nd = 0;
#pragma unroll
    for (int q = 0; q < kPerT; ++q) {
      const int i = tid * kPerT + q;
      if (i < m && key[i] == kc) { ++ct; nd += pos[i] <= pc; }
    }
    if (ct) { atomicAdd(&s_cnt, ct); atomicAdd(&s_need, nd); }
    __syncthreads();
    if (tid == 0) {
      h->pfx = kc;
      h->shift = 0;
      h->cnt_t = s_cnt;
      h->need = s_need;
      h->mode = kWideDone;
    }
    return;
  }
  // large boundary bucket: key range of its members, then radix digits of the order key
  const LinBuckets lb = wide_buckets(h);
  const int d1 = h->d1;
  const int n = h->n;
  const double* s = a.cand_score + qh * a.C1;
  unsigned long long kmx = 0ull, kmn = ~0ull;
  for (int i = tid; i < n; i += 1024) {
    const double v = s[i];
    if (lb.digit(v) == d1) {
      const unsigned long long k = order_key(v);
      kmx = k > kmx ? k : kmx;
      kmn = k < kmn ? k : kmn;
    }
  }
  kmx = cl_block_max_u64(kmx, sm);
  kmn = ~cl_block_max_u64(~kmn, sm);
  unsigned int cnt_b = h->cnt_b;
  unsigned long long mass_b = h->mass_b;
  unsigned long long pfx;
  int shift;
  if (kmx == kmn) {
    pfx = kmx;
    shift = 0;
  } else {
    int hi = 63 - __clzll((long long)(kmx ^ kmn));
    pfx = (hi == 63) ? 0ull : (kmx >> (hi + 1));
    while (true) {
      const int width = (hi + 1) < kDigit ? (hi + 1) : kDigit;
      const int lo = hi + 1 - width;
      cl_clear(sm);
      for (int i = tid; i < n; i += 1024) {
        const double v = s[i];
        if (lb.digit(v) != d1) continue;
        const unsigned long long key = order_key(v);
        if ((hi == 63 ? 0ull : (key >> (hi + 1))) == pfx) {
          const unsigned int bkt = (unsigned int)((key >> lo) & ((1ull << width) - 1));
          atomicAdd(&sm.cnt[bkt], 1u);
          atomicAdd(&sm.mass[bkt], sel_mass(a, v, lb.M));
        }
      }
      const int bstar = cl_boundary<1024, false>(sm, 1, 0, above, tgt, cnt_b, mass_b);
      pfx = (pfx << width) | (unsigned long long)bstar;
      if (cnt_b <= 1 || lo == 0) { shift = lo; break; }
      hi = lo - 1;
    }
  }
  if (tid == 0) {
    h->pfx = pfx;
    h->shift = shift;
    h->cnt_t = cnt_b;
    h->need = need_of(cnt_b, mass_b, tgt, above);
    h->mode = kWideDone;
  }
}

// Keeps (definite and tie) of each chunk.
__global__ void __launch_bounds__(kWideThreads) wide_count_kernel(SelectArgs a, int nch) {
  __shared__ unsigned int red[kWideThreads / 32];
  const int64_t qh = blockIdx.x / nch;
  const int c = (int)(blockIdx.x % nch);
  WideHead* h = wide_head(a, qh);
  if (h->mode == kWideSkip) return;
  const int i0 = c * kWideChunk;
  const int i1 = min(h->n, i0 + kWideChunk);
  const LinBuckets lb = wide_buckets(h);
  const Cutoff cut = wide_cutoff(h);
  const double* s = a.cand_score + qh * a.C1;
  unsigned int nd = 0u, nt = 0u;
#pragma unroll 4
  for (int i = i0 + threadIdx.x; i < i1; i += kWideThreads) {
    const int k = classify(cut, lb, s[i]);
    nd += k == 1;
    nt += k == 2;
  }
  nd = wide_sum<unsigned int, kWideThreads>(nd, red);
  nt = wide_sum<unsigned int, kWideThreads>(nt, red);
  if (threadIdx.x == 0) { wide_chunks(h)[c] = nd; wide_chunks(h)[nch + c] = nt; }
}

// Ordered write: warp w of chunk c's CTA owns a contiguous slice of the chunk.
__global__ void __launch_bounds__(kWideThreads) wide_write_kernel(SelectArgs a, int nch) {
  __shared__ unsigned int wdef[kWideThreads / 32], wtie[kWideThreads / 32];
  __shared__ unsigned long long s_keep_before, s_tie_before, s_total;
  const int64_t qh = blockIdx.x / nch;
  const int c = (int)(blockIdx.x % nch);
  const WideHead* h = wide_head(a, qh);
  if (h->mode == kWideSkip) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int W = kWideThreads / 32;
  const unsigned int lt = (1u << lane) - 1u;
  const Cutoff cut = wide_cutoff(h);
  const bool partial = cut.shift != 64 && cut.cnt_t > 1 && cut.need < cut.cnt_t;
  // keeps and ties of the chunks before this one, and of all of them: warp 0 scans the
  // chunks' counts 32 at a time
  if (warp == 0) {
    unsigned long long keep_run = 0, tie_run = 0;
    for (int base = 0; base < nch; base += 32) {
      const int x = base + lane;
      const unsigned long long t = x < nch ? wide_chunks(h)[nch + x] : 0ull;
      const unsigned long long dd = x < nch ? wide_chunks(h)[x] : 0ull;
      unsigned long long tin = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, tin, o);
        if (lane >= o) tin += y;
      }
      const unsigned long long tie_before_x = tie_run + tin - t;
      unsigned long long take = t;
      if (partial) {
        const long long r = (long long)cut.need - (long long)tie_before_x;
        take = r <= 0 ? 0ull : ((unsigned long long)r < t ? (unsigned long long)r : t);
      }
      const unsigned long long k = dd + take;
      unsigned long long kin = k;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, kin, o);
        if (lane >= o) kin += y;
      }
      if (x == c) { s_keep_before = keep_run + kin - k; s_tie_before = tie_before_x; }
      keep_run += __shfl_sync(0xffffffffu, kin, 31);
      tie_run += __shfl_sync(0xffffffffu, tin, 31);
    }
    if (lane == 0) s_total = keep_run;
  }
  const int i0 = c * kWideChunk;
  const int i1 = min(h->n, i0 + kWideChunk);
  const int len = i1 > i0 ? i1 - i0 : 0;
  const LinBuckets lb = wide_buckets(h);
  const double* s = a.cand_score + qh * a.C1;
  const int* ids = a.cand_ids + qh * a.C1;
  const int C = ((len + W - 1) / W + 31) & ~31;
  const int c0 = i0 + (warp * C < len ? warp * C : len);
  const int c1 = i0 + (warp * C + C < len ? warp * C + C : len);
  unsigned int nd = 0, nt = 0;
  for (int b0 = c0; b0 < c1; b0 += 32) {
    const int i = b0 + lane;
    const int k = i < c1 ? classify(cut, lb, s[i]) : 0;
    nd += __popc(__ballot_sync(0xffffffffu, k == 1));
    nt += __popc(__ballot_sync(0xffffffffu, k == 2));
  }
  if (lane == 0) { wdef[warp] = nd; wtie[warp] = nt; }
  __syncthreads();
  unsigned long long tie_before = s_tie_before, keep_before = s_keep_before;
  for (int w = 0; w < warp; ++w) {
    const unsigned long long t = wtie[w];
    unsigned long long take = t;
    if (partial) {
      const long long r = (long long)cut.need - (long long)tie_before;
      take = r <= 0 ? 0ull : ((unsigned long long)r < t ? (unsigned long long)r : t);
    }
    keep_before += wdef[w] + take;
    tie_before += t;
  }
  long long take = nt;                                   // ties this warp keeps
  if (partial) {
    const long long r = (long long)cut.need - (long long)tie_before;
    take = r <= 0 ? 0 : (r < (long long)nt ? r : (long long)nt);
  }
  unsigned int pos = (unsigned int)keep_before, ties = 0;
  bool overflow = false;
  for (int b0 = c0; b0 < c1; b0 += 32) {
    const int i = b0 + lane;
    const int k = i < c1 ? classify(cut, lb, s[i]) : 0;
    const unsigned int tb = __ballot_sync(0xffffffffu, k == 2);
    const bool keep = k == 1 || (k == 2 && (long long)(ties + __popc(tb & lt)) < take);
    ties += __popc(tb);
    const unsigned int kb = __ballot_sync(0xffffffffu, keep);
    if (keep) emit_kept(a, qh, ids, i, pos + __popc(kb & lt), overflow);
    pos += __popc(kb);
  }
  if (overflow) set_status(a.dev_status, ZHA_ERR_CAPACITY);
  if (c == 0 && tid == 0) {
    const unsigned long long written = s_total;
    a.out_cnt[qh] = (int64_t)written < a.out_cap ? (int)written : a.out_cap;
    int* lc = level_counts(a, qh);
    if (lc) { lc[0] = h->n; lc[1] = (int)written; }
  }
}

static cudaError_t launch_select_wide(const SelectArgs& se, int64_t nqh, int64_t ncap, cudaStream_t s) {
  const int nch = (int)((ncap + kWideChunk - 1) / kWideChunk);
  const unsigned g1 = (unsigned)nqh, gc = (unsigned)(nqh * nch);
  const size_t sort_smem = (size_t)kWideMembers * (2 * sizeof(unsigned long long) + sizeof(int));
  cudaError_t e = cudaFuncSetAttribute(wide_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sort_smem);
  if (e != cudaSuccess) return e;
  if (se.C1 * 8 < (int64_t)(sizeof(WideHead) + 8 * (size_t)nch)) return cudaErrorInvalidValue;   // C1 > 135168
  wide_init_kernel<<<g1, kWideThreads, 0, s>>>(se, nch);
  wide_minmax_kernel<<<gc, kWideThreads, 0, s>>>(se, nch);
  wide_hist_kernel<<<gc, kWideThreads, 0, s>>>(se, nch);
  wide_boundary_kernel<<<g1, 1024, 0, s>>>(se);
  wide_gather_kernel<<<gc, kWideThreads, 0, s>>>(se, nch);
  wide_resolve_kernel<<<g1, 1024, sort_smem, s>>>(se);
  wide_count_kernel<<<gc, kWideThreads, 0, s>>>(se, nch);
  wide_write_kernel<<<gc, kWideThreads, 0, s>>>(se, nch);
  count_launch(7);                                       // with the caller's count: 8
  return cudaGetLastError();
}

static int grid_for(int64_t work, int per_sm) {
  int64_t cap = 148ll * per_sm;
  return (int)(work < cap ? (work < 1 ? 1 : work) : cap);
}

constexpr int kCta1024Cap = 16896;       // candidates a 1024-thread select CTA holds

template <typename K>
static cudaLaunchConfig_t cluster_config(K kernel, cudaLaunchAttribute* attr, int64_t clusters, int cs,
                                         int threads, size_t smem, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cs > 1 ? 1 : 0;                       // a CTA per head: no cluster
  cfg.gridDim = dim3((unsigned)((clusters < 1 ? 1 : clusters) * cs), 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  return cfg;
}

template <typename K>
static cudaError_t launch_cluster(K kernel, const SelectArgs& se, int64_t clusters, int cs, int threads,
                                  size_t smem, cudaStream_t s) {
  if (smem > 0) {
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = cluster_config(kernel, attr, clusters, cs, threads, smem, s);
  return cudaLaunchKernelEx(&cfg, kernel, se);
}

// ---------------------------------------------------------------------------
// The small top levels in one launch.  Levels whose frontier capacity is at most
// kSmallCap nodes (the top of the tree) are scored and selected by one CTA per (sequence,
// query, KV head) unit, level after level: the scores with the arithmetic of
// route_score_kernel (the same fp64 tensor-core products, in the same order), the cutoff
// with the rule of the select kernels (fixed-point masses, target ceil(p Z), order score
// desc then id asc: a candidate is kept iff the mass of the candidates before it is below
// the target), so the kept sets are those of the per-level launches.
// ---------------------------------------------------------------------------

#ifndef ZHA_SMALL_CAP
#define ZHA_SMALL_CAP 64
#endif
constexpr int kSmallCap = ZHA_SMALL_CAP;        // frontier capacity of a fused level
constexpr int kSmallThreads = 256;

struct SmallArgs {
  RouteGeom g;
  int l_lo, l_hi;                                // fused levels: l_hi down to l_lo (>= 2)
  const void* Q;
  const void* k_route[kMaxDepth + 1];            // per level
  const float* b_hat[kMaxDepth + 1];
  double p[kMaxDepth + 1];
  int64_t topk[kMaxDepth + 1];
  int mass_shift;
  int* out_ids;                                  // kept ids of level l_lo, [nqh, out_stride]
  int* out_cnt;
  int64_t out_stride;
  int* level_cnt;                                // nullable [nqh, depth, 2]
  int* level_ids;                                // nullable [nqh, level_ids_stride]
  int64_t level_ids_stride;
  int64_t level_ids_off[kMaxDepth + 1];
  int32_t* dev_status;
};

template <typename KT>
__global__ void __launch_bounds__(kSmallThreads, 2) route_small_kernel(SmallArgs a) {
  __shared__ __align__(16) double qfs[32][32];
  __shared__ double sc[kMaxG][kSmallCap];            // scores of the union's nodes, per head
  __shared__ unsigned long long ms[kMaxG][kSmallCap]; // their fixed-point masses
  __shared__ int uid[kSmallCap];                     // the union of the heads' candidates (ascending)
  __shared__ unsigned int umask[kSmallCap];          // heads that have the union's node as candidate
  __shared__ unsigned int hm[kSmallCap];             // head bits per node id (building the union)
  __shared__ int kept[kMaxG][kSmallCap];             // each head's kept ids (ascending)
  __shared__ int kcnt[kMaxG];
  __shared__ unsigned int wtot[kSmallThreads / 32];
  __shared__ int nu;
  const RouteGeom& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double scale = 1.0 / sqrt((double)kD);
  const int64_t units = (int64_t)g.B * g.nq * g.Hkv;
  const unsigned int all = (g.G >= 32) ? 0xffffffffu : ((1u << g.G) - 1u);
  const int R = g.R;
  constexpr int kVec = 16 / sizeof(KT);
  constexpr int kNv = 32 / kVec;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int64_t bq = u / g.Hkv;
    const int hk = (int)(u % g.Hkv);
    const int64_t b = bq / g.nq;
    const int64_t qh0 = bq * g.Hq + (int64_t)hk * g.G;
    const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
    const int top = pos_ok(g, t) ? top_level(g, t) : 0;
    __syncthreads();                                     // shared memory of the previous unit
    if (!pos_ok(g, t) && tid == 0) set_status(a.dev_status, ZHA_ERR_INVALID_ARG);
    // fused levels above the query's top level: empty selections
    if (a.level_cnt && tid < g.G)
      for (int l = a.l_hi; l >= a.l_lo && l > top; --l) {
        int* lc = a.level_cnt + ((qh0 + tid) * g.depth + (l - 1)) * 2;
        lc[0] = 0;
        lc[1] = 0;
      }
    if (top < a.l_lo) continue;                          // the per-level launches start at its top
    for (int i = tid; i < 32 * 32; i += kSmallThreads) {
      const int s2 = i / 32, L = i % 32, h = L >> 2;
      const KT* q = reinterpret_cast<const KT*>(a.Q) + qh0 * kD;
      qfs[s2][L] = h < g.G ? to_f64(q[h * kD + 32 * (L & 3) + s2]) : 0.0;
    }
    for (int l = top < a.l_hi ? top : a.l_hi; l >= a.l_lo; --l) {
      const int64_t nvis = visible_nodes(t, g.span[l]);  // <= n_cap(l) <= kSmallCap
      const bool at_top = l == top;
      const int64_t orph_lo = at_top ? 0 : visible_nodes(t, g.span[l + 1]) * g.branch;
      // ---- the union of the heads' candidates with their head bits
      for (int i = tid; i < kSmallCap; i += kSmallThreads) hm[i] = 0u;
      __syncthreads();
      if (at_top) {
        for (int i = tid; i < nvis; i += kSmallThreads) hm[i] = all;
      } else {
        for (int h = warp; h < g.G; h += kSmallThreads / 32)
          for (int k = lane; k < kcnt[h] * g.branch; k += 32) {
            const int id = kept[h][k / g.branch] * g.branch + k % g.branch;
            if (id < kSmallCap) atomicOr(&hm[id], 1u << h);
          }
        for (int64_t i = orph_lo + tid; i < nvis; i += kSmallThreads) hm[i] = all;
      }
      __syncthreads();
      {
        const bool on = tid < kSmallCap && hm[tid] != 0u;
        const unsigned int bal = __ballot_sync(0xffffffffu, on);
        if (lane == 0) wtot[warp] = __popc(bal);
        __syncthreads();
        unsigned int before = __popc(bal & ((1u << lane) - 1u));
        for (int w = 0; w < warp; ++w) before += wtot[w];
        if (on) { uid[before] = tid; umask[before] = hm[tid]; }
        if (tid == 0) {
          unsigned int tot = 0;
          for (int w = 0; w < kSmallThreads / 32; ++w) tot += wtot[w];
          nu = (int)tot;
        }
      }
      __syncthreads();
      // ---- scores: groups of 8 union nodes x 8 heads on the fp64 tensor cores
      const int64_t node0 = (b * g.Hkv + hk) * g.ncap[l];
      const int h0 = 2 * (lane & 3), h1 = h0 + 1;
      for (int grp = warp; grp * 8 < nu; grp += kSmallThreads / 32) {
        const int pos = grp * 8 + (lane >> 2);
        const bool has = pos < nu;
        const int id = has ? uid[pos] : 0;
        const unsigned int m = has ? umask[pos] : 0u;
        double best0 = -INFINITY, best1 = -INFINITY;
        for (int r0 = 0; r0 < R; r0 += 4) {
          // the rows of up to four references load together (one memory latency per four)
          constexpr int kRb = 4;
          uint4 v[kRb][kNv];
          float bh[kRb];
#pragma unroll
          for (int rr = 0; rr < kRb; ++rr) {
            const bool on = m && r0 + rr < R;
            const uint4* src = reinterpret_cast<const uint4*>(
                reinterpret_cast<const KT*>(a.k_route[l]) + ((node0 + id) * R + r0 + rr) * kD + 32 * (lane & 3));
#pragma unroll
            for (int i = 0; i < kNv; ++i) v[rr][i] = on ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
            bh[rr] = on ? __ldg(a.b_hat[l] + (node0 + id) * R + r0 + rr) : 0.f;
          }
#pragma unroll
          for (int rr = 0; rr < kRb; ++rr) {
            if (r0 + rr >= R) break;
            double c0[4] = {0.0, 0.0, 0.0, 0.0}, c1[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
            for (int s2 = 0; s2 < 32; ++s2) {
              const double av = (double)u4_elem<KT>(v[rr][s2 / kVec], s2 % kVec);
              mma_f64(c0[s2 & 3], c1[s2 & 3], av, qfs[s2][lane]);
            }
            const double bb = (double)bh[rr];
            best0 = fmax(best0, fma((c0[0] + c0[1]) + (c0[2] + c0[3]), scale, bb));
            best1 = fmax(best1, fma((c1[0] + c1[1]) + (c1[2] + c1[3]), scale, bb));
          }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int h = q ? h1 : h0;
          if (h < g.G && ((m >> h) & 1u)) {
            double s = q ? best1 : best0;
            if (s == 0.0) s = 0.0;                       // one zero (no -0.0) for the key order
            sc[h][pos] = s;
          }
        }
      }
      __syncthreads();
      // ---- the cutoff of each head (warp h)
      if (warp < g.G) {
        const int h = warp;
        const int64_t qh = qh0 + h;
        const unsigned int hb = 1u << h;
        int n_h = 0;
        double M = -INFINITY;
        for (int i = lane; i < nu; i += 32)
          if (umask[i] & hb) { ++n_h; M = fmax(M, sc[h][i]); }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          n_h += __shfl_xor_sync(0xffffffffu, n_h, o);
          M = fmax(M, __shfl_xor_sync(0xffffffffu, M, o));
        }
        unsigned long long Z = 0;
        for (int i = lane; i < nu; i += 32)
          if (umask[i] & hb) {
            const unsigned long long e = a.topk[l] > 0 ? 1ull : mass_of(sc[h][i], M, a.mass_shift);
            ms[h][i] = e;
            Z += e;
          }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
        __syncwarp();
        const bool keep_all = n_h == 0 || (a.topk[l] > 0 ? a.topk[l] >= n_h : a.p[l] >= 1.0);
        unsigned long long tgt = 0;
        if (!keep_all)
          tgt = a.topk[l] > 0 ? ((unsigned long long)a.topk[l] < Z ? (unsigned long long)a.topk[l] : Z)
                              : target_of(a.p[l], Z);
        int kc = 0;
        for (int base = 0; base < nu; base += 32) {
          const int i = base + lane;
          bool keep = false;
          if (i < nu && (umask[i] & hb)) {
            keep = keep_all;
            if (!keep) {
              const double si = sc[h][i];
              unsigned long long before = 0;             // mass of the candidates ordered before i
              for (int j = 0; j < nu; ++j)
                if ((umask[j] & hb) && (sc[h][j] > si || (sc[h][j] == si && j < i))) before += ms[h][j];
              keep = before < tgt;
            }
          }
          const unsigned int bal = __ballot_sync(0xffffffffu, keep);
          if (keep) {
            const int at = kc + __popc(bal & ((1u << lane) - 1u));
            const int id = uid[i];
            kept[h][at] = id;
            if (a.level_ids) a.level_ids[qh * a.level_ids_stride + a.level_ids_off[l] + at] = id;
            if (l == a.l_lo) a.out_ids[qh * a.out_stride + at] = id;
          }
          kc += __popc(bal);
        }
        if (lane == 0) {
          kcnt[h] = kc;
          if (a.level_cnt) {
            int* lc = a.level_cnt + (qh * g.depth + (l - 1)) * 2;
            lc[0] = n_h;
            lc[1] = kc;
          }
          if (l == a.l_lo) a.out_cnt[qh] = kc;
        }
      }
      __syncthreads();
    }
  }
}

#ifndef ZHA_WARP_SELECT_MAX
#define ZHA_WARP_SELECT_MAX 256
#endif

// One select launch per level.  Kernels, by the frontier capacity ncap they hold:
//   warp     a warp per head (scores in shared memory)            ncap <= 1024
//   cta256   a CTA of 256 threads per head (30 or 48 KiB)         ncap <= 2560 or 4096
//   cta1024  a CTA of 1024 threads per head (198 KiB)             ncap <= 16896
//   cluster  2 / 4 / 8 CTAs of 1024 threads per head              ncap <= 8 * 16896
//   wide     a chain of grid-wide kernels over (head, chunk)      above
// The widest kernel whose resident heads (148 SMs x CTAs per SM) cover every head of the
// level runs them in one wave at the lowest latency per head; when none does, the
// narrowest one that holds ncap takes the most heads at once.
static cudaError_t launch_select(const SelectArgs& se, int64_t nqh, int64_t ncap, cudaStream_t s) {
  const int64_t res256 = 148ll * 3, res1024 = 148;
  int kind;                                            // 0 warp, 1 cta256, 2 cta1024, 3 cluster, 4 wide
  if (ncap <= ZHA_WARP_SELECT_MAX) kind = 0;           // small frontiers: a warp per head is the quickest
  else if (ncap <= kCta1024Cap && nqh <= res1024) kind = 2;
  else if (ncap <= 4096 && nqh <= res256) kind = 1;
  else if (ncap <= kWarpCap) kind = 0;
  else if (ncap <= 4096) kind = 1;
  else if (ncap <= kCta1024Cap) kind = 2;
  else if (ncap <= 8ll * kCta1024Cap) kind = 3;
  else kind = 4;
  if (kind == 0) {
    const size_t smem = sizeof(WarpSelSmem);
    cudaError_t e = cudaFuncSetAttribute(route_select_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    route_select_warp_kernel<<<grid_for((nqh + kWarpSelWarps - 1) / kWarpSelWarps, 3), kWarpSelWarps * 32, smem,
                               s>>>(se);
    return cudaGetLastError();
  }
  if (kind == 1 && ncap <= 2560)                       // 56 KiB per CTA: 4 resident per SM
    return launch_cluster(route_select_block_kernel<256, 2560, false>, se, nqh < 4 * 148 ? nqh : 4 * 148, 1,
                          256, 2560 * (sizeof(double) + sizeof(int)), s);
  if (kind == 1)
    return launch_cluster(route_select_block_kernel<256, 4096, false>, se, nqh < res256 ? nqh : res256, 1, 256,
                          4096 * (sizeof(double) + sizeof(int)), s);
  if (kind == 2)
    return launch_cluster(route_select_block_kernel<1024, kCta1024Cap, false>, se, nqh < res1024 ? nqh : res1024,
                          1, 1024, kCta1024Cap * (sizeof(double) + sizeof(int)), s);
  if (kind == 3) {
    const int cs = ncap <= 2 * kCta1024Cap ? 2 : ncap <= 4 * kCta1024Cap ? 4 : 8;
    const int64_t per = 148 / cs;
    return launch_cluster(route_select_block_kernel<1024, kCta1024Cap, true>, se, nqh < per ? nqh : per, cs,
                          1024, kCta1024Cap * (sizeof(double) + sizeof(int)), s);
  }
  return launch_select_wide(se, nqh, ncap, s);
}

// ---------------------------------------------------------------------------
// host side: the launches of one routing call
// ---------------------------------------------------------------------------



static RouteGeom make_route_geom(const zha_geom& g, int nq, const int64_t* q_pos, int64_t pu) {
  RouteGeom r{};
  r.B = g.B; r.nq = nq; r.Hq = g.Hq; r.Hkv = g.Hkv; r.G = g.Hq / g.Hkv; r.R = g.R;
  r.branch = g.branch; r.depth = g.depth; r.q_pos = q_pos; r.pos_uniform = pu; r.t_cap = g.t_cap;
  for (int l = 1; l <= g.depth; ++l) { r.span[l] = span_of(g, l); r.ncap[l] = ncap_of(g, l); }
  r.span[g.depth + 1] = r.span[g.depth] * g.branch;
  r.ncap[g.depth + 1] = 0;
  return r;
}

static int mass_shift_for(int64_t n) {
  int bits = 0;
  while ((1ll << bits) <= n) ++bits;     // bits to hold n
  return 62 - bits;
}


template <typename KT>
static cudaError_t route_levels(const RouteCall& c) {
  const zha_geom& g = *c.g;
  const TreeLayout L = tree_layout(g);
  const RouteWs w = route_ws(g, c.nq, 0);
  const RouteGeom rg = make_route_geom(g, c.nq, c.q_pos, c.pos_uniform);
  const int64_t nqh = (int64_t)g.B * c.nq * g.Hq;
  int* selbuf[2] = {(int*)(c.ws + w.selA), (int*)(c.ws + w.selB)};
  int* selcnt[2] = {(int*)(c.ws + w.selA_cnt), (int*)(c.ws + w.selB_cnt)};
  int64_t level_ids_stride = 0;
  for (int l = 2; l <= g.depth; ++l) level_ids_stride += ncap_of(g, l);
  int64_t level_off = level_ids_stride;
  // One position for every query (a decode step) and no level counts requested: the levels
  // above the query's top level hold no visible node, so their launches are skipped (they
  // would only record empty selections).  Level 1 always runs: it writes the leaf counts.
  int lmax = g.depth;
  if (!c.q_pos && !c.level_cnt && !c.level_ids && c.pos_uniform >= 0 && c.pos_uniform < g.t_cap) {
    const int64_t vis = (c.pos_uniform / kLeaf) * kLeaf;
    int top = 0;
    for (int l = g.depth; l >= 1 && top == 0; --l)
      if (vis / span_of(g, l) >= 1) top = l;
    lmax = top < 1 ? 1 : top;
  }
  for (int l = g.depth; l > lmax; --l)
    if (l >= 2) level_off -= ncap_of(g, l);
  // the top levels whose frontier capacity is at most kSmallCap: one fused launch
  int l_lo = lmax + 1;
  for (int l = lmax; l >= 2 && ncap_of(g, l) <= kSmallCap; --l) l_lo = l;
  if (l_lo <= lmax) {
    SmallArgs sm{};
    sm.g = rg; sm.l_lo = l_lo; sm.l_hi = lmax; sm.Q = c.Q;
    int64_t off = 0;
    for (int l = 2; l <= g.depth; ++l) { sm.level_ids_off[l] = off; off += ncap_of(g, l); }
    for (int l = l_lo; l <= lmax; ++l) {
      sm.k_route[l] = (char*)c.tree + L.lv[l].k_route_off;
      sm.b_hat[l] = (const float*)((char*)c.tree + L.lv[l].b_hat_off);
      sm.p[l] = c.p_levels ? c.p_levels[l - 1] : c.p;
      sm.topk[l] = c.k_levels ? c.k_levels[l - 1] : 0;
    }
    sm.mass_shift = mass_shift_for(w.C1);
    sm.out_ids = selbuf[l_lo & 1]; sm.out_cnt = selcnt[l_lo & 1]; sm.out_stride = w.C2;
    sm.level_cnt = c.level_cnt; sm.level_ids = c.level_ids; sm.level_ids_stride = level_ids_stride;
    sm.dev_status = c.dev_status;
    const int64_t units = (int64_t)g.B * c.nq * g.Hkv;
    trace_begin(ZHA_TRACE_ROUTE_FUSED, c.stream);
    route_small_kernel<KT><<<grid_for(units, 4), kSmallThreads, 0, c.stream>>>(sm);
    trace_end(ZHA_TRACE_ROUTE_FUSED, c.stream);
    count_launch();
    cudaError_t e = launch_status("route_small_kernel");
    if (e != cudaSuccess) return e;
    for (int l = lmax; l >= l_lo; --l) level_off -= ncap_of(g, l);
    lmax = l_lo - 1;
  }
  for (int l = lmax; l >= 1; --l) {
    const int cur = l & 1, prev = (l + 1) & 1;
    ScoreArgs sa{};
    sa.g = rg; sa.level = l; sa.Q = c.Q;
    sa.k_route = (char*)c.tree + L.lv[l].k_route_off;
    sa.b_hat = (const float*)((char*)c.tree + L.lv[l].b_hat_off);
    sa.parents = selbuf[prev]; sa.parents_cnt = selcnt[prev];
    sa.C1 = w.C1; sa.C2 = w.C2;
    sa.cand_ids = (int*)(c.ws + w.cand_ids);
    sa.cand_score = (double*)(c.ws + w.cand_score);
    sa.cand_cnt = (int*)(c.ws + w.cand_cnt);
    sa.dev_status = c.dev_status;
    {
      const int64_t per_blk = kScoreSlots / g.branch;
      int64_t nb = (L.lv[l].n_cap + kScoreSlots - 1) / kScoreSlots;
      if (l < g.depth) {
        const int64_t nbp = (L.lv[l + 1].n_cap + per_blk - 1) / per_blk + 1;
        if (nbp > nb) nb = nbp;
      }
      sa.nblk = nb < 1 ? 1 : nb;
    }
    const int64_t units = (int64_t)g.B * c.nq * g.Hkv;
    trace_begin(ZHA_TRACE_ROUTE_SCORE, c.stream);
    if (units * sa.nblk <= 2 * 148)                      // few items: shortest chains
      route_score_kernel<KT, 1><<<grid_for(units * sa.nblk, 1), kScoreSlots * 4, 0, c.stream>>>(sa);
    else
      route_score_kernel<KT, 4><<<grid_for(units * sa.nblk, 8), kScoreSlots, 0, c.stream>>>(sa);
    trace_end(ZHA_TRACE_ROUTE_SCORE, c.stream);
    count_launch();
    cudaError_t e = launch_status("route_score_kernel");
    if (e != cudaSuccess) return e;

    SelectArgs se{};
    se.g = rg; se.level = l; se.flat = 0; se.p = c.p_levels ? c.p_levels[l - 1] : c.p;
    se.topk = c.k_levels ? c.k_levels[l - 1] : 0;
    se.mass_shift = mass_shift_for(w.C1);
    se.cand_ids = sa.cand_ids; se.cand_score = sa.cand_score;
    se.cand_mass = (unsigned long long*)(c.ws + w.cand_mass);
    se.cand_cnt = sa.cand_cnt; se.C1 = w.C1;
    if (l == 1) {
      se.out_ids = c.leaf_ids; se.out_cnt = c.leaf_cnt; se.out_stride = c.leaf_cap; se.out_cap = c.leaf_cap;
    } else {
      se.out_ids = selbuf[cur]; se.out_cnt = selcnt[cur]; se.out_stride = w.C2; se.out_cap = (int)w.C2;
    }
    se.level_cnt = c.level_cnt;
    se.level_ids = c.level_ids;
    se.level_ids_stride = level_ids_stride;
    if (l >= 2) level_off -= ncap_of(g, l);
    se.level_ids_off = l >= 2 ? level_off : 0;
    se.level_ids_cap = l >= 2 ? ncap_of(g, l) : 0;
    se.dev_status = c.dev_status;
    trace_begin(ZHA_TRACE_ROUTE_SELECT, c.stream);
    e = launch_select(se, nqh, L.lv[l].n_cap, c.stream);
    count_launch();
    if (e != cudaSuccess) { note_cuda_error(e, "route select"); return e; }
    trace_end(ZHA_TRACE_ROUTE_SELECT, c.stream);
  }
  return cudaSuccess;
}

cudaError_t route_all(const RouteCall& c) {
  return c.g->dtype == ZHA_BF16 ? route_levels<__nv_bfloat16>(c) : route_levels<float>(c);
}

template <typename KT>
static cudaError_t flat_select_t(const RouteCall& c) {
  const zha_geom& g = *c.g;
  const RouteWs w = route_ws(g, c.nq, 0);
  const RouteGeom rg = make_route_geom(g, c.nq, c.q_pos, c.pos_uniform);
  const int64_t units = (int64_t)g.B * c.nq * g.Hkv;
  const int64_t nqh = (int64_t)g.B * c.nq * g.Hq;
  FlatArgs fa{};
  fa.g = rg; fa.Q = c.Q; fa.K = c.tree; fa.t_cap = g.t_cap; fa.C1 = w.C1;
  fa.cand_ids = (int*)(c.ws + w.cand_ids);
  fa.cand_score = (double*)(c.ws + w.cand_score);
  fa.cand_cnt = (int*)(c.ws + w.cand_cnt);
  fa.nblk = (w.C1 + 7) / 8;
  if (fa.nblk < 1) fa.nblk = 1;
  cudaError_t e;
  if (g.dtype == ZHA_BF16) {                           // tensor cores, K streamed by TMA
    trace_begin(ZHA_TRACE_ROUTE_SCORE, c.stream);
    e = flat_tc_launch(g, c.nq, c.Q, c.tree, c.q_pos, c.pos_uniform, w.C1, fa.cand_ids, fa.cand_score,
                       fa.cand_cnt, c.dev_status, c.stream);
    trace_end(ZHA_TRACE_ROUTE_SCORE, c.stream);
    count_launch();
    if (e != cudaSuccess) return e;
    e = launch_status("flat_tc_kernel");
  } else {
    flat_score_kernel<KT><<<grid_for(units * fa.nblk, 8), 256, 0, c.stream>>>(fa);
    count_launch();
    e = launch_status("flat_score_kernel");
  }
  if (e != cudaSuccess) return e;
  SelectArgs se{};
  se.g = rg; se.level = 1; se.flat = 1; se.p = c.p;
  se.mass_shift = mass_shift_for(w.C1);
  se.cand_ids = fa.cand_ids; se.cand_score = fa.cand_score;
  se.cand_mass = (unsigned long long*)(c.ws + w.cand_mass);
  se.cand_cnt = fa.cand_cnt; se.C1 = w.C1;
  se.out_ids = c.leaf_ids; se.out_cnt = c.leaf_cnt; se.out_stride = c.leaf_cap; se.out_cap = c.leaf_cap;
  se.dev_status = c.dev_status;
  e = launch_select(se, nqh, w.C1, c.stream);
  count_launch();
  if (e != cudaSuccess) note_cuda_error(e, "route select (flat)");
  return e;
}

// Flat indexer: `c.tree` carries the K cache pointer.
cudaError_t flat_select(const RouteCall& c) {
  return c.g->dtype == ZHA_BF16 ? flat_select_t<__nv_bfloat16>(c) : flat_select_t<float>(c);
}

}  // namespace zha
