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

constexpr int kScoreThreads = 128;

template <typename KT>
__global__ void __launch_bounds__(kScoreThreads) route_score_kernel(ScoreArgs a) {
  __shared__ __align__(16) double qfs[32][32];
  __shared__ int rank[kScoreThreads][kMaxG];     // per parent slot: rank in each head's list
  __shared__ int pcnt[kMaxG];
  const RouteGeom& g = a.g;
  const int tid = threadIdx.x;
  const int64_t units = (int64_t)g.B * g.nq * g.Hkv;
  const double scale = 1.0 / sqrt((double)kD);
  const int per_blk = kScoreThreads / g.branch;          // parents per work item
  for (int64_t w = blockIdx.x; w < units * a.nblk; w += gridDim.x) {
    const int64_t u = w / a.nblk;
    const int64_t blk = w % a.nblk;
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
      if (blk * kScoreThreads >= nvis) continue;
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
    // B fragments of the mma: qfs[s][L] = q[head L/4][32 * (L%4) + s] (0 for heads >= G)
    for (int i = tid; i < 32 * 32; i += kScoreThreads) {
      const int s2 = i / 32, L = i % 32, h = L >> 2;
      const KT* q = reinterpret_cast<const KT*>(a.Q) + qh0 * kD;
      qfs[s2][L] = h < g.G ? to_f64(q[h * kD + 32 * (L & 3) + s2]) : 0.0;
    }
    __syncthreads();
    if (blk == 0 && tid < g.G)
      a.cand_cnt[qh0 + tid] = (int)(at_top ? nvis : (int64_t)pcnt[tid] * g.branch + (nvis - orph_lo));
    if (mode == 3) continue;
    if (mode == 1) {
      // rank of each parent of this item in each head's kept list (-1: not kept)
      for (int i = tid; i < per_blk * g.G; i += kScoreThreads) {
        const int j = i / g.G, h = i % g.G;
        const int64_t p = blk * per_blk + j;
        int r = -1;
        if (p < npar) {
          const int* lst = a.parents + (qh0 + h) * a.C2;
          int lo = 0, hi = pcnt[h];
          while (lo < hi) { const int m = (lo + hi) >> 1; if (lst[m] < p) lo = m + 1; else hi = m; }
          if (lo < pcnt[h] && lst[lo] == p) r = lo;
        }
        rank[j][h] = r;
      }
      __syncthreads();
    }
    // Scores on the fp64 tensor cores: each warp takes its 32 slots as 4 groups of 8
    // nodes; D[8 nodes x 8 heads] += A[8 nodes x 4 dims] . B[4 dims x 8 heads] per
    // mma.m8n8k4.f64.  Lane L holds A[node L/4][dim 32*(L%4) + s] and B[dim][head L/4]
    // at k-step s (qf[s][L] in shared memory), so each lane reads 32 contiguous dims of
    // its node's row.  The (group, reference) steps are software-pipelined: the next
    // step's row is in flight while the current step's 32 mma run.
    const int lane = tid & 31, warp = tid >> 5;
    const int h0 = 2 * (lane & 3), h1 = h0 + 1;         // this lane's heads in D
    // node of this lane's row in group grp, and the heads that have it as a candidate
    auto slot_of = [&](int grp, int64_t& id, unsigned int& mask, int& j, int& c) {
      const int slot = warp * 32 + grp * 8 + (lane >> 2);
      mask = 0;
      j = 0;
      c = 0;
      if (mode == 0) {
        id = blk * kScoreThreads + slot;
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
    unsigned int any_mask = 0;
    for (int grp = 0; grp < 4; ++grp) {
      int64_t id; unsigned int m; int jj, cc;
      slot_of(grp, id, m, jj, cc);
      any_mask |= m;
    }
    if (!__any_sync(0xffffffffu, any_mask != 0)) continue;   // warp-uniform
    constexpr int kVec = 16 / sizeof(KT);
    constexpr int kNv = 32 / kVec;                       // 16-byte vectors of 32 dims
    const int R = g.R;
    const int nsteps = 4 * R;                            // even
    const int64_t node0 = (b * g.Hkv + hk) * g.ncap[a.level];
    auto load_step = [&](uint4 (&v)[kNv], int st) {
      const int grp = st / R, r = st - grp * R;
      int64_t id; unsigned int m; int jj, cc;
      slot_of(grp, id, m, jj, cc);
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const KT*>(a.k_route) + ((node0 + id) * R + r) * kD + 32 * (lane & 3));
#pragma unroll
      for (int i = 0; i < kNv; ++i) v[i] = m ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    };
    double best0 = -INFINITY, best1 = -INFINITY;
    auto compute_step = [&](const uint4 (&v)[kNv], int st) {
      const int grp = st / R, r = st - grp * R;
      double ca0 = 0.0, ca1 = 0.0, cb0 = 0.0, cb1 = 0.0;
#pragma unroll
      for (int s2 = 0; s2 < 32; ++s2) {
        const double av = (double)u4_elem<KT>(v[s2 / kVec], s2 % kVec);  // exact widening
        const double qv = qfs[s2][lane];
        if (s2 & 1) mma_f64(cb0, cb1, av, qv);
        else mma_f64(ca0, ca1, av, qv);
      }
      int64_t id; unsigned int m; int jj, cc;
      slot_of(grp, id, m, jj, cc);
      const double bb = m ? (double)a.b_hat[(node0 + id) * R + r] : 0.0;
      best0 = fmax(best0, fma(ca0 + cb0, scale, bb));
      best1 = fmax(best1, fma(ca1 + cb1, scale, bb));
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
    uint4 vA[kNv], vB[kNv];
    load_step(vA, 0);
    for (int st = 0; st < nsteps; st += 2) {
      load_step(vB, st + 1);
      compute_step(vA, st);
      if (st + 2 < nsteps) load_step(vA, st + 2);
      compute_step(vB, st + 1);
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
// top-p select over one level's candidates: exact radix select on the fp64 order key
// with fixed-point masses (a warp per query head up to kWarpSelMax candidates, a
// cluster of CTAs per query head above)
// ---------------------------------------------------------------------------

constexpr int kWarpSelMax = 1024;        // larger frontiers use the cluster kernel
constexpr int kDigit = 11;
constexpr int kBuckets = 1 << kDigit;

struct SelectArgs {
  RouteGeom g;
  int level;
  int flat;                      // 1: a single level over all visible leaves
  double p;
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
// warp select: one warp per query head for frontiers of up to kWarpSelMax candidates
// (the common case): 8-bit digits, per-warp histograms in shared memory and warp
// shuffles for every reduction and scan.
// ---------------------------------------------------------------------------

constexpr int kWarpSelWarps = 8;
constexpr int kWDigit = 8;
constexpr int kWBuckets = 1 << kWDigit;

struct WarpSelSmem {
  unsigned int cnt[kWarpSelWarps][kWBuckets];
  unsigned long long mass[kWarpSelWarps][kWBuckets];
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

__global__ void __launch_bounds__(kWarpSelWarps * 32) route_select_warp_kernel(SelectArgs a) {
  __shared__ WarpSelSmem sm;
  const RouteGeom& g = a.g;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned int* hcnt = sm.cnt[wid];
  unsigned long long* hmass = sm.mass[wid];
  const int64_t nqh = (int64_t)g.B * g.nq * g.Hq;
  for (int64_t qh = (int64_t)blockIdx.x * kWarpSelWarps + wid; qh < nqh;
       qh += (int64_t)gridDim.x * kWarpSelWarps) {
    const int64_t bq = qh / g.Hq;
    const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
    const int top = !pos_ok(g, t) ? 0 : a.flat ? (visible_nodes(t, kLeaf) >= 1 ? 1 : 0) : top_level(g, t);
    int* lc = a.level_cnt ? a.level_cnt + (qh * g.depth + (a.level - 1)) * 2 : nullptr;
    if (a.level > top) {
      if (lane == 0) {
        if (lc) { lc[0] = 0; lc[1] = 0; }
        if (a.level == 1) a.out_cnt[qh] = 0;
      }
      continue;
    }
    const int n = a.cand_cnt[qh];
    if (n > kWarpSelMax) continue;                      // the cluster kernel takes it
    const double* s = a.cand_score + qh * a.C1;
    const int* ids = a.cand_ids + qh * a.C1;
    unsigned long long* E = a.cand_mass + qh * a.C1;
    // 1. maximum and minimum
    // every pass walks the candidates 8 per lane at a time, loads first (in flight together)
#define WSEL_BATCH(LOADS, BODY)                                                     \
    for (int base_ = 0; base_ < n; base_ += 32 * 8) {                               \
      _Pragma("unroll") for (int u_ = 0; u_ < 8; ++u_) {                            \
        const int i = base_ + u_ * 32 + lane;                                       \
        LOADS                                                                       \
      }                                                                             \
      _Pragma("unroll") for (int u_ = 0; u_ < 8; ++u_) {                            \
        const int i = base_ + u_ * 32 + lane;                                       \
        if (i < n) { BODY }                                                         \
      }                                                                             \
    }
    double sv[8];
    unsigned long long ev[8];
    double mx = -INFINITY, mn = INFINITY;
    WSEL_BATCH({ sv[u_] = i < n ? s[i] : 0.0; }, { mx = fmax(mx, sv[u_]); mn = fmin(mn, sv[u_]); })
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmax(mx, shfl_xor_f64(mx, o));
      mn = fmin(mn, shfl_xor_f64(mn, o));
    }
    // 2. fixed-point masses and their exact total
    unsigned long long z = 0;
    WSEL_BATCH({ sv[u_] = i < n ? s[i] : 0.0; }, {
      const unsigned long long e = __double2ull_rn(ldexp(exp(sv[u_] - mx), a.mass_shift));
      E[i] = e;
      z += e;
    })
    const unsigned long long Z = warp_sum_u64(z);
    __syncwarp();
    // 3. cutoff
    const bool keep_all = a.p >= 1.0 || n == 0;
    unsigned long long pfx = 0, need = 0;
    int shift = 0;
    if (!keep_all) {
      double tg = ceil(a.p * (double)Z);
      unsigned long long tgt = tg < 1.0 ? 1ull : (unsigned long long)tg;
      if (tgt > Z) tgt = Z;
      const unsigned long long kmax = order_key(mx), kmin = order_key(mn);
      unsigned long long above = 0;
      unsigned int cnt_b = (unsigned int)n;
      unsigned long long mass_b = Z;
      if (kmax == kmin) {
        pfx = kmax;
      } else {
        int hi = 63 - __clzll((long long)(kmax ^ kmin));
        pfx = (hi == 63) ? 0ull : (kmax >> (hi + 1));
        while (true) {
          const int width = (hi + 1) < kWDigit ? (hi + 1) : kWDigit;
          const int lo = hi + 1 - width;
#pragma unroll
          for (int q = 0; q < kWBuckets / 32; ++q) { hcnt[lane + 32 * q] = 0; hmass[lane + 32 * q] = 0; }
          __syncwarp();
          WSEL_BATCH({ sv[u_] = i < n ? s[i] : 0.0; ev[u_] = i < n ? E[i] : 0ull; }, {
            const unsigned long long key = order_key(sv[u_]);
            if ((hi == 63 ? 0ull : (key >> (hi + 1))) == pfx) {
              const unsigned int bkt = (unsigned int)((key >> lo) & ((1ull << width) - 1));
              atomicAdd(&hcnt[bkt], 1u);
              atomicAdd(&hmass[bkt], ev[u_]);
            }
          })
          __syncwarp();
          // lane L owns the 8 buckets below kWBuckets - 8L (from the top: highest scores)
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
          bstar = __shfl_sync(0xffffffffu, bstar, src);
          above = __shfl_sync(0xffffffffu, above_new, src);
          cnt_b = hcnt[bstar];
          mass_b = hmass[bstar];
          pfx = (pfx << width) | (unsigned long long)bstar;
          __syncwarp();
          if (cnt_b <= 1 || lo == 0) { shift = lo; break; }
          hi = lo - 1;
        }
      }
      if (cnt_b <= 1) {
        need = 1;
      } else {
        const unsigned long long e1 = mass_b / cnt_b;
        need = e1 == 0 ? cnt_b : (tgt - above + e1 - 1) / e1;
        if (need < 1) need = 1;
        if (need > cnt_b) need = cnt_b;
      }
    }
    // 4. ordered compaction: lane L owns the contiguous candidates [L*per, (L+1)*per)
    const int per = (n + 31) / 32;
    const int i0 = lane * per, i1 = (i0 + per < n) ? i0 + per : n;
    unsigned int nt = 0;
    if (!keep_all) {
#pragma unroll 8
      for (int i = i0; i < i1; ++i) nt += (order_key(s[i]) >> shift) == pfx;
    }
    unsigned int tie_total;
    unsigned int tie_rank = warp_excl_scan(nt, &tie_total);
    unsigned int nk = 0;
    {
      unsigned int tr = tie_rank;
#pragma unroll 8
      for (int i = i0; i < i1; ++i) {
        bool keep = keep_all;
        if (!keep_all) {
          const unsigned long long kk = order_key(s[i]) >> shift;
          keep = kk > pfx || (kk == pfx && tr++ < need);
        }
        nk += keep;
      }
    }
    unsigned int written;
    unsigned int pos = warp_excl_scan(nk, &written);
    int* outp = a.out_ids + qh * a.out_stride;
    bool overflow = false;
#pragma unroll 4
    for (int i = i0; i < i1; ++i) {
      bool keep = keep_all;
      if (!keep_all) {
        const unsigned long long kk = order_key(s[i]) >> shift;
        keep = kk > pfx || (kk == pfx && tie_rank++ < need);
      }
      if (keep) {
        const int id = ids[i];
        if ((int64_t)pos < a.out_cap) outp[pos] = id;
        else overflow = true;
        if (a.level_ids && a.level >= 2 && (int64_t)pos < a.level_ids_cap)
          a.level_ids[qh * a.level_ids_stride + a.level_ids_off + pos] = id;
        ++pos;
      }
    }
    if (overflow) set_status(a.dev_status, ZHA_ERR_CAPACITY);
    if (lane == 0) {
      a.out_cnt[qh] = (int64_t)written < a.out_cap ? (int)written : a.out_cap;
      if (lc) { lc[0] = n; lc[1] = (int)written; }
    }
    __syncwarp();
  }
#undef WSEL_BATCH
}

// ---------------------------------------------------------------------------
// cluster select: one thread-block cluster (1..8 CTAs of kClThreads) per query head, for
// frontiers above kWarpSelMax.  Each CTA takes a contiguous slice of the candidates; the
// cluster's rank-0 CTA sums the per-CTA maxima, totals and digit histograms through
// distributed shared memory and publishes every decision back into each CTA, so all CTAs
// take identical decisions.  Cluster barriers are hardware barriers (no spin loops).
// ---------------------------------------------------------------------------

constexpr int kClThreads = 512;
constexpr int kClMaxCta = 8;

struct ClSmem {
  unsigned int cnt[kBuckets];
  unsigned long long mass[kBuckets];
  unsigned long long wsum[kClThreads / 32];
  double wd[kClThreads / 32];
  unsigned int wcnt[kClThreads / 32];
  // per-CTA contributions, written into the rank-0 CTA by every rank
  unsigned long long slot_kmax[kClMaxCta], slot_kmin[kClMaxCta], slot_z[kClMaxCta];
  unsigned int slot_tie[kClMaxCta], slot_keep[kClMaxCta];
  // decisions published by rank 0
  unsigned long long d_above, d_mass_b;
  unsigned int d_cnt_b;
  int d_bstar;
};

__device__ __forceinline__ double cl_block_max(double v, ClSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, shfl_xor_f64(v, o));
  __syncthreads();
  if (lane == 0) sm.wd[warp] = v;
  __syncthreads();
  double r = sm.wd[0];
  for (int i = 1; i < kClThreads / 32; ++i) r = fmax(r, sm.wd[i]);
  return r;
}

__device__ __forceinline__ unsigned long long cl_block_sum(unsigned long long v, ClSmem& sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sm.wsum[warp] = v;
  __syncthreads();
  unsigned long long r = 0;
  for (int i = 0; i < kClThreads / 32; ++i) r += sm.wsum[i];
  return r;
}

__device__ __forceinline__ unsigned int cl_excl_scan(unsigned int v, ClSmem& sm, unsigned int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) sm.wcnt[warp] = x;
  __syncthreads();
  unsigned int before = 0, all = 0;
  for (int i = 0; i < kClThreads / 32; ++i) {
    if (i < warp) before += sm.wcnt[i];
    all += sm.wcnt[i];
  }
  *total = all;
  return before + x - v;
}

__global__ void __launch_bounds__(kClThreads) route_select_cluster_kernel(SelectArgs a) {
  __shared__ ClSmem sm;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int cr = (int)cluster.block_rank();
  ClSmem* lead = cluster.map_shared_rank(&sm, 0);
  const RouteGeom& g = a.g;
  const int tid = threadIdx.x;
  const int64_t nqh = (int64_t)g.B * g.nq * g.Hq;
  const int64_t nclusters = gridDim.x / CS;
  for (int64_t qh = blockIdx.x / CS; qh < nqh; qh += nclusters) {
    const int64_t bq = qh / g.Hq;
    const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
    const int top = !pos_ok(g, t) ? 0 : a.flat ? (visible_nodes(t, kLeaf) >= 1 ? 1 : 0) : top_level(g, t);
    if (a.level > top) continue;                         // the warp kernel writes the counts
    const int n = a.cand_cnt[qh];
    if (n <= kWarpSelMax) continue;                      // the warp kernel takes it
    int* lc = a.level_cnt ? a.level_cnt + (qh * g.depth + (a.level - 1)) * 2 : nullptr;
    const double* s = a.cand_score + qh * a.C1;
    const int* ids = a.cand_ids + qh * a.C1;
    unsigned long long* E = a.cand_mass + qh * a.C1;
    const int chunk = (n + CS - 1) / CS;
    const int r0 = cr * chunk < n ? cr * chunk : n;
    const int r1 = r0 + chunk < n ? r0 + chunk : n;

    // 1. maximum and minimum over the cluster
    double mx = -INFINITY, mn = INFINITY;
    for (int i = r0 + tid; i < r1; i += kClThreads) { const double v = s[i]; mx = fmax(mx, v); mn = fmin(mn, v); }
    mx = cl_block_max(mx, sm);
    mn = -cl_block_max(-mn, sm);
    if (tid == 0) {
      lead->slot_kmax[cr] = r1 > r0 ? order_key(mx) : 0ull;
      lead->slot_kmin[cr] = r1 > r0 ? order_key(mn) : ~0ull;
    }
    cluster.sync();
    unsigned long long kmax = 0, kmin = ~0ull;
    for (int r = 0; r < CS; ++r) {
      const unsigned long long x = lead->slot_kmax[r], y = lead->slot_kmin[r];
      kmax = x > kmax ? x : kmax;
      kmin = y < kmin ? y : kmin;
    }
    // back from the order key to the score
    const unsigned long long mb = (kmax >> 63) ? (kmax & 0x7fffffffffffffffull) : ~kmax;
    const double M = __longlong_as_double((long long)mb);
    // 2. fixed-point masses and their exact total
    unsigned long long z = 0;
    for (int i = r0 + tid; i < r1; i += kClThreads) {
      const unsigned long long e = __double2ull_rn(ldexp(exp(s[i] - M), a.mass_shift));
      E[i] = e;
      z += e;
    }
    z = cl_block_sum(z, sm);
    if (tid == 0) lead->slot_z[cr] = z;
    cluster.sync();
    unsigned long long Z = 0;
    for (int r = 0; r < CS; ++r) Z += lead->slot_z[r];

    // 3. cutoff, with identical decisions in every CTA
    const bool keep_all = a.p >= 1.0;
    unsigned long long pfx = 0, need = 0;
    int shift = 0;
    if (!keep_all) {
      double tg = ceil(a.p * (double)Z);
      unsigned long long tgt = tg < 1.0 ? 1ull : (unsigned long long)tg;
      if (tgt > Z) tgt = Z;
      unsigned long long above = 0, mass_b = Z;
      unsigned int cnt_b = (unsigned int)n;
      if (kmax == kmin) {
        pfx = kmax;
      } else {
        int hi = 63 - __clzll((long long)(kmax ^ kmin));
        pfx = (hi == 63) ? 0ull : (kmax >> (hi + 1));
        while (true) {
          const int width = (hi + 1) < kDigit ? (hi + 1) : kDigit;
          const int lo = hi + 1 - width;
          for (int i = tid; i < kBuckets; i += kClThreads) { sm.cnt[i] = 0; sm.mass[i] = 0; }
          __syncthreads();
          for (int i = r0 + tid; i < r1; i += kClThreads) {
            const unsigned long long key = order_key(s[i]);
            if ((hi == 63 ? 0ull : (key >> (hi + 1))) == pfx) {
              const unsigned int bkt = (unsigned int)((key >> lo) & ((1ull << width) - 1));
              atomicAdd(&sm.cnt[bkt], 1u);
              atomicAdd(&sm.mass[bkt], E[i]);
            }
          }
          cluster.sync();                                // every CTA's histogram is complete
          if (cr == 0) {
            // sum the CTAs' histograms (rank order) and find the boundary bucket
            constexpr int kPer = kBuckets / kClThreads;
            unsigned long long bm[kPer];
            unsigned int bc[kPer];
            unsigned long long local = 0;
#pragma unroll
            for (int q = 0; q < kPer; ++q) {
              const int bkt = kBuckets - 1 - (tid * kPer + q);
              unsigned long long m2 = 0;
              unsigned int c2 = 0;
              for (int r = 0; r < CS; ++r) {
                ClSmem* o = cluster.map_shared_rank(&sm, r);
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
                    ClSmem* o = cluster.map_shared_rank(&sm, r);
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
          cluster.sync();                                // decision published; histograms free
          const int bstar = sm.d_bstar;
          above = sm.d_above;
          cnt_b = sm.d_cnt_b;
          mass_b = sm.d_mass_b;
          pfx = (pfx << width) | (unsigned long long)bstar;
          if (cnt_b <= 1 || lo == 0) { shift = lo; break; }
          hi = lo - 1;
        }
      }
      if (cnt_b <= 1) {
        need = 1;
      } else {
        const unsigned long long e1 = mass_b / cnt_b;
        need = e1 == 0 ? cnt_b : (tgt - above + e1 - 1) / e1;
        if (need < 1) need = 1;
        if (need > cnt_b) need = cnt_b;
      }
    }

    // 4. ordered compaction: thread t of CTA r owns a contiguous piece of the CTA's slice
    const int len = r1 - r0;
    const int per = (len + kClThreads - 1) / kClThreads;
    const int i0 = r0 + tid * per < r1 ? r0 + tid * per : r1;
    const int i1 = i0 + per < r1 ? i0 + per : r1;
    unsigned int nt = 0;
    if (!keep_all)
      for (int i = i0; i < i1; ++i) nt += (order_key(s[i]) >> shift) == pfx;
    unsigned int tie_cta;
    unsigned int tie_rank = cl_excl_scan(nt, sm, &tie_cta);
    if (tid == 0) lead->slot_tie[cr] = tie_cta;
    cluster.sync();
    for (int r = 0; r < cr; ++r) tie_rank += lead->slot_tie[r];
    unsigned int nk = 0;
    {
      unsigned int tr = tie_rank;
      for (int i = i0; i < i1; ++i) {
        bool keep = keep_all;
        if (!keep_all) {
          const unsigned long long kk = order_key(s[i]) >> shift;
          keep = kk > pfx || (kk == pfx && tr++ < need);
        }
        nk += keep;
      }
    }
    unsigned int keep_cta;
    unsigned int pos = cl_excl_scan(nk, sm, &keep_cta);
    if (tid == 0) lead->slot_keep[cr] = keep_cta;
    cluster.sync();
    unsigned int written = 0;
    for (int r = 0; r < CS; ++r) {
      const unsigned int k = lead->slot_keep[r];
      if (r < cr) pos += k;
      written += k;
    }
    int* outp = a.out_ids + qh * a.out_stride;
    bool overflow = false;
    for (int i = i0; i < i1; ++i) {
      bool keep = keep_all;
      if (!keep_all) {
        const unsigned long long kk = order_key(s[i]) >> shift;
        keep = kk > pfx || (kk == pfx && tie_rank++ < need);
      }
      if (keep) {
        const int id = ids[i];
        if ((int64_t)pos < a.out_cap) outp[pos] = id;
        else overflow = true;
        if (a.level_ids && a.level >= 2 && (int64_t)pos < a.level_ids_cap)
          a.level_ids[qh * a.level_ids_stride + a.level_ids_off + pos] = id;
        ++pos;
      }
    }
    if (overflow) set_status(a.dev_status, ZHA_ERR_CAPACITY);
    if (cr == 0 && tid == 0) {
      a.out_cnt[qh] = (int64_t)written < a.out_cap ? (int)written : a.out_cap;
      if (lc) { lc[0] = n; lc[1] = (int)written; }
    }
    cluster.sync();                                      // slots and smem reused by the next head
  }
}

static cudaError_t launch_select_cluster(const SelectArgs& se, int64_t nqh, int64_t ncap, cudaStream_t s) {
  int cs = (int)((ncap + 8191) / 8192);
  cs = cs < 1 ? 1 : (cs > kClMaxCta ? kClMaxCta : (cs > 4 ? 8 : (cs > 2 ? 4 : cs)));
  int64_t clusters = nqh < (2 * 148) / cs ? nqh : (2 * 148) / cs;
  if (clusters < 1) clusters = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(clusters * cs), 1, 1);
  cfg.blockDim = dim3(kClThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, route_select_cluster_kernel, se);
}

// ---------------------------------------------------------------------------
// host driver
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

static int grid_for(int64_t work, int per_sm) {
  int64_t cap = 148ll * per_sm;
  return (int)(work < cap ? (work < 1 ? 1 : work) : cap);
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
  for (int l = g.depth; l >= 1; --l) {
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
      const int64_t per_blk = kScoreThreads / g.branch;
      int64_t nb = (L.lv[l].n_cap + kScoreThreads - 1) / kScoreThreads;
      if (l < g.depth) {
        const int64_t nbp = (L.lv[l + 1].n_cap + per_blk - 1) / per_blk + 1;
        if (nbp > nb) nb = nbp;
      }
      sa.nblk = nb < 1 ? 1 : nb;
    }
    const int64_t units = (int64_t)g.B * c.nq * g.Hkv;
    trace_begin(ZHA_TRACE_ROUTE_SCORE, c.stream);
    route_score_kernel<KT><<<grid_for(units * sa.nblk, 8), kScoreThreads, 0, c.stream>>>(sa);
    trace_end(ZHA_TRACE_ROUTE_SCORE, c.stream);
    count_launch();
    cudaError_t e = launch_status("route_score_kernel");
    if (e != cudaSuccess) return e;

    SelectArgs se{};
    se.g = rg; se.level = l; se.flat = 0; se.p = c.p;
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
    route_select_warp_kernel<<<grid_for((nqh + kWarpSelWarps - 1) / kWarpSelWarps, 8), kWarpSelWarps * 32, 0,
                               c.stream>>>(se);
    count_launch();
    e = launch_status("route_select_warp_kernel");
    if (e != cudaSuccess) return e;
    if (L.lv[l].n_cap > kWarpSelMax) {                   // frontiers too large for one warp
      e = launch_select_cluster(se, nqh, L.lv[l].n_cap, c.stream);
      count_launch();
      if (e != cudaSuccess) { note_cuda_error(e, "route_select_cluster_kernel"); return e; }
    }
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
  flat_score_kernel<KT><<<grid_for(units * fa.nblk, 8), 256, 0, c.stream>>>(fa);
  count_launch();
  cudaError_t e = launch_status("flat_score_kernel");
  if (e != cudaSuccess) return e;
  SelectArgs se{};
  se.g = rg; se.level = 1; se.flat = 1; se.p = c.p;
  se.mass_shift = mass_shift_for(w.C1);
  se.cand_ids = fa.cand_ids; se.cand_score = fa.cand_score;
  se.cand_mass = (unsigned long long*)(c.ws + w.cand_mass);
  se.cand_cnt = fa.cand_cnt; se.C1 = w.C1;
  se.out_ids = c.leaf_ids; se.out_cnt = c.leaf_cnt; se.out_stride = c.leaf_cap; se.out_cap = c.leaf_cap;
  se.dev_status = c.dev_status;
  route_select_warp_kernel<<<grid_for((nqh + kWarpSelWarps - 1) / kWarpSelWarps, 8), kWarpSelWarps * 32, 0,
                             c.stream>>>(se);
  count_launch();
  e = launch_status("route_select_warp_kernel(flat)");
  if (e != cudaSuccess) return e;
  if (w.C1 > kWarpSelMax) {
    e = launch_select_cluster(se, nqh, w.C1, c.stream);
    count_launch();
    if (e != cudaSuccess) { note_cuda_error(e, "route_select_cluster_kernel(flat)"); return e; }
  }
  return launch_status("route_select_cluster_kernel(flat)");
}

// Flat indexer: `c.tree` carries the K cache pointer.
cudaError_t flat_select(const RouteCall& c) {
  return c.g->dtype == ZHA_BF16 ? flat_select_t<__nv_bfloat16>(c) : flat_select_t<float>(c);
}

}  // namespace zha
