// Sparse attention over I(q) = {0} u (chunks of S_1(q)) u C_cur(q) ("ZHA summary" page,
// Routing), the dense flash-decode baseline, and their shared plumbing.
//
// The G query heads of one KV head share one gather: for each (b, query, KV head) unit
// the heads' ascending leaf lists are merged into a union of chunk ids, each with a
// bit mask of the heads that selected it.  The union is built per block of kRange chunk
// ids (no global zeroing, one pass), split into work items of `cps` entries, and a
// persistent kernel walks the items: each item streams its K/V blocks once and keeps
// an online softmax (m, l, o[d]) per head; a combine kernel merges the items' partials
// by log-sum-exp (split-KV partials, arXiv 2610.42112 App. D-B1).
#include <type_traits>

#include "zha_internal.cuh"

namespace zha {

struct AttnGeom {
  int B, nq, Hq, Hkv, G;
  int64_t t_cap;
  const int64_t* q_pos;
  int64_t pos_uniform;
  int64_t nr, cps;               // ranges per unit, chunks per split
};

// ---------------------------------------------------------------------------
// union of the heads' chunk lists, one CTA per (unit, range of kRange chunk ids)
// Entry ids: -1 = the first key alone (the sink), n_vis = the query's own chunk
// [V(t), t], otherwise a full leaf chunk.
// ---------------------------------------------------------------------------

struct UnionArgs {
  AttnGeom g;
  int dense;
  const int* leaf_ids;           // [B, nq, Hq, leaf_cap]
  const int* leaf_cnt;
  int leaf_cap;
  int* stage_ids;                // [pairs, kRange + 2]
  unsigned int* stage_mask;
  int* stage_cnt;                // [pairs]
  int32_t* dev_status;
};

__global__ void __launch_bounds__(256) union_kernel(UnionArgs a) {
  __shared__ unsigned int mask[kRange];
  __shared__ unsigned int wtot[8];
  __shared__ unsigned int sink_mask;
  const AttnGeom& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pair = blockIdx.x;
  const int64_t u = pair / g.nr;
  const int64_t r = pair % g.nr;
  const int64_t bq = u / g.Hkv;
  const int hk = (int)(u % g.Hkv);
  const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
  if (t < 0 || t >= g.t_cap) {                       // rejected position: nothing to attend
    if (tid == 0) { a.stage_cnt[pair] = 0; if (r == 0) set_status(a.dev_status, ZHA_ERR_INVALID_ARG); }
    return;
  }
  const int64_t nvis = visible_nodes(t, kLeaf);
  const int64_t lo = r * kRange, hi = lo + kRange;
  const unsigned int full = (g.G >= 32) ? 0xffffffffu : ((1u << g.G) - 1u);
  for (int i = tid; i < kRange; i += 256) mask[i] = 0;
  if (tid == 0) sink_mask = 0;
  __syncthreads();
  if (a.dense) {
    for (int64_t i = lo + tid; i < hi && i < nvis; i += 256) mask[i - lo] = full;
  } else {
    // each head's slice [lower_bound(lo), lower_bound(hi)) of its ascending list, then
    // one flat pass over all slices so that every thread's loads are independent
    __shared__ int s_b0[kMaxG], s_off[kMaxG + 1];
    if (warp < g.G) {
      // warp h finds its head's slice of its ascending list
      const int64_t qh = bq * g.Hq + hk * g.G + warp;
      const int* lst = a.leaf_ids + qh * a.leaf_cap;
      int cnt = a.leaf_cnt[qh];
      if (cnt > a.leaf_cap) cnt = a.leaf_cap;
      if (cnt < 0) cnt = 0;
      const int x0 = warp_lower_bound(lst, cnt, lo);
      const int x1 = warp_lower_bound(lst, cnt, hi);
      if (lane == 0) {
        s_b0[warp] = x0;
        s_off[warp + 1] = x1 - x0;
      }
    }
    __syncthreads();
    if (tid == 0) {
      s_off[0] = 0;
      for (int h = 0; h < g.G; ++h) s_off[h + 1] += s_off[h];
    }
    __syncthreads();
    const int total_ids = s_off[g.G];
    int h = 0;                                    // i only grows: the head index follows it
#pragma unroll 8
    for (int i = tid; i < total_ids; i += 256) {
      while (i >= s_off[h + 1]) ++h;
      const int64_t qh = bq * g.Hq + hk * g.G + h;
      const int id = a.leaf_ids[qh * a.leaf_cap + s_b0[h] + (i - s_off[h])];
      // ids outside [lo, hi) mean an unsorted list; outside [0, nvis) an invisible chunk
      if (id < lo || id >= hi || id >= nvis) { set_status(a.dev_status, ZHA_ERR_INVALID_ARG); continue; }
      atomicOr(&mask[id - lo], 1u << h);
    }
  }
  __syncthreads();
  // the first key: heads that did not select chunk 0 still attend to key 0
  if (!a.dense && r == 0 && nvis >= 1 && tid == 0) sink_mask = full & ~mask[0];
  __syncthreads();
  // compaction in id order; the sink entry goes first, the partial chunk last
  int* out_ids = a.stage_ids + pair * (kRange + 2);
  unsigned int* out_mask = a.stage_mask + pair * (kRange + 2);
  unsigned int base = 0;
  if (sink_mask) {
    if (tid == 0) { out_ids[0] = -1; out_mask[0] = sink_mask; }
    base = 1;
  }
  constexpr int kPer = kRange / 256;     // consecutive ids per thread
  unsigned int cntl = 0;
  for (int q = 0; q < kPer; ++q) cntl += mask[tid * kPer + q] != 0;
  unsigned int x = cntl;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  unsigned int before = base, total = base;
  for (int i = 0; i < 8; ++i) { if (i < warp) before += wtot[i]; total += wtot[i]; }
  before += x - cntl;
  for (int q = 0; q < kPer; ++q) {
    const int i = tid * kPer + q;
    if (mask[i]) { out_ids[before] = (int)(lo + i); out_mask[before] = mask[i]; ++before; }
  }
  if (tid == 0) {
    if (nvis >= lo && nvis < hi) { out_ids[total] = (int)nvis; out_mask[total] = full; ++total; }
    a.stage_cnt[pair] = (int)total;
  }
}

// Work items: ceil(stage_cnt / cps) per (unit, range) pair; exclusive offsets in pair_off.
__global__ void __launch_bounds__(1024) plan_kernel(const int* stage_cnt, int64_t pairs, int64_t cps,
                                                    int* pair_off) {
  __shared__ unsigned int wtot[32];
  __shared__ unsigned int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < pairs; base += 1024) {
    const int64_t i = base + tid;
    const unsigned int v = i < pairs ? (unsigned int)((stage_cnt[i] + cps - 1) / cps) : 0u;
    unsigned int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wtot[warp] = x;
    __syncthreads();
    unsigned int before = carry, tot = 0;
    for (int w = 0; w < 32; ++w) { if (w < warp) before += wtot[w]; tot += wtot[w]; }
    if (i < pairs) pair_off[i] = (int)(before + x - v);
    __syncthreads();
    if (tid == 0) carry += tot;
    __syncthreads();
  }
  if (tid == 0) pair_off[pairs] = (int)carry;
}

// ---------------------------------------------------------------------------
// split-KV attention, CUDA-core version (any dtype, G <= 8): 256 threads, warp h <-> head h
// ---------------------------------------------------------------------------

struct AttnArgs {
  AttnGeom g;
  const void* Q;
  const void* K;
  const void* V;
  const int* stage_ids;
  const unsigned int* stage_mask;
  const int* stage_cnt;
  const int* pair_off;
  int64_t pairs;
  float* partials;               // [items, G, kPartStride]: o[d], m, l
};

constexpr int kRowPad = kD + 4;   // fp32 smem row stride (16-byte aligned, bank-skewed)

__device__ __forceinline__ int64_t find_pair(const int* off, int64_t pairs, int64_t item) {
  int64_t lo = 0, hi = pairs;             // last pair with off[pair] <= item
  while (hi - lo > 1) { const int64_t m = (lo + hi) >> 1; if (off[m] <= item) lo = m; else hi = m; }
  return lo;
}

template <typename KT>
__global__ void __launch_bounds__(256) attn_split_kernel(AttnArgs a) {
  extern __shared__ __align__(16) float smf[];
  float* Ks = smf;                         // [64][kRowPad]
  float* Vs = Ks + kLeaf * kRowPad;        // [64][kRowPad]
  float* Qs = Vs + kLeaf * kRowPad;        // [kMaxG][kD]
  const AttnGeom& g = a.g;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float sl2 = 1.4426950408889634f / sqrtf((float)kD);   // log2(e) / sqrt(d)
  const int64_t total_items = a.pair_off[a.pairs];
  for (int64_t item = blockIdx.x; item < total_items; item += gridDim.x) {
    const int64_t pair = find_pair(a.pair_off, a.pairs, item);
    const int64_t sub = item - a.pair_off[pair];
    const int64_t u = pair / g.nr;
    const int64_t bq = u / g.Hkv;
    const int hk = (int)(u % g.Hkv);
    const int64_t b = bq / g.nq;
    const int64_t t = query_pos(g.q_pos, g.pos_uniform, bq);
    const int64_t vstart = (t / kLeaf) * kLeaf;
    const int64_t nvis = vstart / kLeaf;
    const int cnt = a.stage_cnt[pair];
    const int e0 = (int)(sub * g.cps);
    const int e1 = (int)((sub + 1) * g.cps < cnt ? (sub + 1) * g.cps : cnt);
    __syncthreads();
    for (int i = tid; i < g.G * kD; i += 256)
      Qs[i] = to_f32(reinterpret_cast<const KT*>(a.Q)[(bq * g.Hq + hk * g.G) * kD + i]);
    const KT* Kb = reinterpret_cast<const KT*>(a.K) + (b * g.Hkv + hk) * g.t_cap * kD;
    const KT* Vb = reinterpret_cast<const KT*>(a.V) + (b * g.Hkv + hk) * g.t_cap * kD;
    float m = -INFINITY, l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    const int h = warp;
    for (int e = e0; e < e1; ++e) {
      const int id = a.stage_ids[pair * (kRange + 2) + e];
      const unsigned int msk = a.stage_mask[pair * (kRange + 2) + e];
      int64_t k0;
      int len;
      if (id < 0) { k0 = 0; len = 1; }
      else if (id == nvis) { k0 = vstart; len = (int)(t - vstart + 1); }
      else { k0 = (int64_t)id * kLeaf; len = kLeaf; }
      __syncthreads();
      constexpr int kVec = 16 / sizeof(KT);
      constexpr int kRowVec = kD / kVec;
      for (int i = tid; i < len * kRowVec; i += 256) {
        const int row = i / kRowVec, c = (i % kRowVec) * kVec;
        const uint4 kv = *reinterpret_cast<const uint4*>(Kb + (k0 + row) * kD + c);
        const uint4 vv = *reinterpret_cast<const uint4*>(Vb + (k0 + row) * kD + c);
        const KT* ke = reinterpret_cast<const KT*>(&kv);
        const KT* ve = reinterpret_cast<const KT*>(&vv);
#pragma unroll
        for (int x = 0; x < kVec; ++x) {
          Ks[row * kRowPad + c + x] = to_f32(ke[x]);
          Vs[row * kRowPad + c + x] = to_f32(ve[x]);
        }
      }
      __syncthreads();
      if (h < g.G && ((msk >> h) & 1u)) {
        // scores of keys lane and lane + 32, in log2 units
        float s0 = 0.f, s1 = 0.f;
        const float4* q4 = reinterpret_cast<const float4*>(Qs + h * kD);
        const float4* ka = reinterpret_cast<const float4*>(Ks + lane * kRowPad);
        const float4* kb = reinterpret_cast<const float4*>(Ks + (lane + 32) * kRowPad);
#pragma unroll 8
        for (int c = 0; c < kD / 4; ++c) {
          const float4 qv = q4[c], x = ka[c], y = kb[c];
          s0 = fmaf(qv.x, x.x, fmaf(qv.y, x.y, fmaf(qv.z, x.z, fmaf(qv.w, x.w, s0))));
          s1 = fmaf(qv.x, y.x, fmaf(qv.y, y.y, fmaf(qv.z, y.z, fmaf(qv.w, y.w, s1))));
        }
        s0 = lane < len ? s0 * sl2 : -INFINITY;
        s1 = lane + 32 < len ? s1 * sl2 : -INFINITY;
        float mx = fmaxf(s0, s1);
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
        const float mnew = fmaxf(m, mx);
        const float alpha = exp2f(m - mnew);          // m = -inf at start -> 0
        const float p0 = exp2f(s0 - mnew), p1 = exp2f(s1 - mnew);
        float ps = p0 + p1;
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, x);
        l = l * alpha + ps;
        o.x *= alpha; o.y *= alpha; o.z *= alpha; o.w *= alpha;
        for (int j = 0; j < len; ++j) {
          const float pj = __shfl_sync(0xffffffffu, j < 32 ? p0 : p1, j & 31);
          const float4 vv = reinterpret_cast<const float4*>(Vs + j * kRowPad)[lane];
          o.x = fmaf(pj, vv.x, o.x); o.y = fmaf(pj, vv.y, o.y);
          o.z = fmaf(pj, vv.z, o.z); o.w = fmaf(pj, vv.w, o.w);
        }
        m = mnew;
      }
    }
    if (h < g.G) {
      float* P = a.partials + ((int64_t)item * g.G + h) * kPartStride;
      reinterpret_cast<float4*>(P)[lane] = o;
      if (lane == 0) { P[kD] = m; P[kD + 1] = l; }
    }
  }
}

// ---------------------------------------------------------------------------
// combine: one CTA of 128 threads per (unit, head); thread <-> dim
// ---------------------------------------------------------------------------

// Combine of the split partials (log-sum-exp of (o, m, l) per head, fixed orders, so the
// result is deterministic).  Units of at most kCombBlock items: combine_warp_kernel; larger
// ones: combine_cta_kernel over blocks of kCtaItems items (one block: the output directly;
// several: block partials, then combine_cta_blocks_kernel over the blocks).
constexpr int kCombBlock = 128;
constexpr int kCtaItems = 512;

// Combine for units of at most kCombBlock items (the common case): one CTA per unit, warp
// h <-> head h, lane <-> 4 dims.  Two passes in item order: the maximum M of the partials'
// m, then L = sum 2^(m_i - M) l_i and o = sum 2^(m_i - M) o_i with every load independent
// of the running state (deterministic, fixed order).
template <typename OT>
__global__ void __launch_bounds__(kMaxG * 32) combine_warp_kernel(AttnGeom g, const int* pair_off,
                                                                const float* partials, OT* O, float* lse) {
  const int64_t u = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (h >= g.G) return;
  const int64_t i0 = pair_off[u * g.nr], i1 = pair_off[(u + 1) * g.nr];
  float M = -INFINITY;
  for (int64_t i = i0 + lane; i < i1; i += 32) M = fmaxf(M, partials[(i * g.G + h) * kPartStride + kD]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
#pragma unroll 4
    for (int64_t i = i0; i < i1; ++i) {
      const float* P = partials + (i * g.G + h) * kPartStride;
      const float4 o4 = *reinterpret_cast<const float4*>(P + 4 * lane);
      const float w = exp2f(P[kD] - M);                  // 0 for an empty partial (m = -inf)
      L = fmaf(w, P[kD + 1], L);
      acc.x = fmaf(w, o4.x, acc.x);
      acc.y = fmaf(w, o4.y, acc.y);
      acc.z = fmaf(w, o4.z, acc.z);
      acc.w = fmaf(w, o4.w, acc.w);
    }
  }
  const int64_t bq = u / g.Hkv;
  const int hk = (int)(u % g.Hkv);
  const int64_t qh = bq * g.Hq + hk * g.G + h;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  OT* out = O + qh * kD + 4 * lane;
  out[0] = from_f32<OT>(acc.x * inv);
  out[1] = from_f32<OT>(acc.y * inv);
  out[2] = from_f32<OT>(acc.z * inv);
  out[3] = from_f32<OT>(acc.w * inv);
  if (lse && lane == 0) lse[qh] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

// One CTA of 8 warps per (unit, head, block of kCtaItems items): the block's maximum M first,
// then warp w sums the items w, w + 8, ... (lane <-> 4 dims) and the eight warp sums are
// added in warp order.
template <typename OT>
__global__ void __launch_bounds__(256) combine_cta_kernel(AttnGeom g, const int* pair_off, float* partials,
                                                        int64_t nbl, OT* O, float* lse) {
  __shared__ float wm[8], wl[8];
  __shared__ float4 wacc[8][32];
  const int64_t uh = blockIdx.x / nbl, blk = blockIdx.x % nbl;
  const int64_t u = uh / g.G;
  const int h = (int)(uh % g.G);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t i0 = pair_off[u * g.nr], i1 = pair_off[(u + 1) * g.nr];
  const int64_t b0 = i0 + blk * kCtaItems;
  if (b0 >= i1 && blk > 0) return;                   // uniform over the CTA
  const int64_t b1 = b0 + kCtaItems < i1 ? b0 + kCtaItems : i1;
  float M = -INFINITY;
  for (int64_t i = b0 + tid; i < b1; i += 256) M = fmaxf(M, partials[(i * g.G + h) * kPartStride + kD]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) wm[warp] = M;
  __syncthreads();
  M = wm[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) M = fmaxf(M, wm[w]);
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
#pragma unroll 4
    for (int64_t i = b0 + warp; i < b1; i += 8) {
      const float* P = partials + (i * g.G + h) * kPartStride;
      const float4 o4 = *reinterpret_cast<const float4*>(P + 4 * lane);
      const float w = exp2f(P[kD] - M);
      L = fmaf(w, P[kD + 1], L);
      acc.x = fmaf(w, o4.x, acc.x);
      acc.y = fmaf(w, o4.y, acc.y);
      acc.z = fmaf(w, o4.z, acc.z);
      acc.w = fmaf(w, o4.w, acc.w);
    }
  }
  wacc[warp][lane] = acc;
  if (lane == 0) wl[warp] = L;
  __syncthreads();
  if (warp != 0) return;
  L = 0.f;
  acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    L += wl[w];
    const float4 a4 = wacc[w][lane];
    acc.x += a4.x; acc.y += a4.y; acc.z += a4.z; acc.w += a4.w;
  }
  if (i1 - i0 > kCtaItems) {
    // the block's (o, m, l) replaces its first partial (every read of the block is done)
    float* P = partials + (b0 * g.G + h) * kPartStride;
    *reinterpret_cast<float4*>(P + 4 * lane) = acc;
    if (lane == 0) { P[kD] = M; P[kD + 1] = L; }
    return;
  }
  const int64_t bq = u / g.Hkv;
  const int hk = (int)(u % g.Hkv);
  const int64_t qh = bq * g.Hq + hk * g.G + h;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  OT* out = O + qh * kD + 4 * lane;
  out[0] = from_f32<OT>(acc.x * inv);
  out[1] = from_f32<OT>(acc.y * inv);
  out[2] = from_f32<OT>(acc.z * inv);
  out[3] = from_f32<OT>(acc.w * inv);
  if (lse && lane == 0) lse[qh] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

// Second stage for units of more than kCtaItems items: one warp per (unit, head) merges the
// block partials (at items i0, i0 + kCtaItems, ...) in block order, two passes as above.
template <typename OT>
__global__ void __launch_bounds__(kMaxG * 32) combine_cta_blocks_kernel(AttnGeom g, const int* pair_off,
                                                                      const float* partials, OT* O, float* lse) {
  const int64_t u = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (h >= g.G) return;
  const int64_t i0 = pair_off[u * g.nr], i1 = pair_off[(u + 1) * g.nr];
  if (i1 - i0 <= kCtaItems) return;                  // written by the first stage
  float M = -INFINITY;
  for (int64_t b = i0 + (int64_t)lane * kCtaItems; b < i1; b += 32ll * kCtaItems)
    M = fmaxf(M, partials[(b * g.G + h) * kPartStride + kD]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY) {
    for (int64_t b = i0; b < i1; b += kCtaItems) {
      const float* P = partials + (b * g.G + h) * kPartStride;
      const float4 o4 = *reinterpret_cast<const float4*>(P + 4 * lane);
      const float w = exp2f(P[kD] - M);
      L = fmaf(w, P[kD + 1], L);
      acc.x = fmaf(w, o4.x, acc.x);
      acc.y = fmaf(w, o4.y, acc.y);
      acc.z = fmaf(w, o4.z, acc.z);
      acc.w = fmaf(w, o4.w, acc.w);
    }
  }
  const int64_t bq = u / g.Hkv;
  const int hk = (int)(u % g.Hkv);
  const int64_t qh = bq * g.Hq + hk * g.G + h;
  const float inv = L > 0.f ? 1.f / L : 0.f;
  OT* out = O + qh * kD + 4 * lane;
  out[0] = from_f32<OT>(acc.x * inv);
  out[1] = from_f32<OT>(acc.y * inv);
  out[2] = from_f32<OT>(acc.z * inv);
  out[3] = from_f32<OT>(acc.w * inv);
  if (lse && lane == 0) lse[qh] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side: the launches of one attention call
// ---------------------------------------------------------------------------



template <typename KT>
static cudaError_t attention_t(const AttnCall& c) {
  const zha_geom& g = *c.g;
  const AttnWs w = attn_ws(g, c.nq, 0, c.cps);
  AttnGeom ag{};
  ag.B = g.B; ag.nq = c.nq; ag.Hq = g.Hq; ag.Hkv = g.Hkv; ag.G = g.Hq / g.Hkv; ag.t_cap = g.t_cap;
  ag.q_pos = c.q_pos; ag.pos_uniform = c.pos_uniform; ag.nr = w.nr; ag.cps = w.cps;

  UnionArgs ua{};
  ua.g = ag; ua.dense = c.dense; ua.leaf_ids = c.leaf_ids; ua.leaf_cnt = c.leaf_cnt;
  ua.leaf_cap = c.leaf_cap;
  ua.stage_ids = (int*)(c.ws + w.stage_ids);
  ua.stage_mask = (unsigned int*)(c.ws + w.stage_mask);
  ua.stage_cnt = (int*)(c.ws + w.stage_cnt);
  ua.dev_status = c.dev_status;
  union_kernel<<<(unsigned)w.pairs, 256, 0, c.stream>>>(ua);
  count_launch();
  cudaError_t e = launch_status("union_kernel");
  if (e != cudaSuccess) return e;

  int* pair_off = (int*)(c.ws + w.pair_off);
  plan_kernel<<<1, 1024, 0, c.stream>>>(ua.stage_cnt, w.pairs, w.cps, pair_off);
  count_launch();
  if ((e = launch_status("plan_kernel")) != cudaSuccess) return e;

  AttnArgs aa{};
  aa.g = ag; aa.Q = c.Q; aa.K = c.K; aa.V = c.V;
  aa.stage_ids = ua.stage_ids; aa.stage_mask = ua.stage_mask; aa.stage_cnt = ua.stage_cnt;
  aa.pair_off = pair_off; aa.pairs = w.pairs;
  aa.partials = (float*)(c.ws + w.partials);
  if (std::is_same<KT, __nv_bfloat16>::value) {
    // bf16 caches: TMA-fed, tensor-core kernel (zha_attn_tc.cu)
    trace_begin(ZHA_TRACE_ATTN, c.stream);
    e = attn_tc_launch(c, w, aa.stage_ids, aa.stage_mask, aa.stage_cnt, pair_off, aa.partials);
    trace_end(ZHA_TRACE_ATTN, c.stream);
    count_launch();
    if (e != cudaSuccess) return e;
    if ((e = launch_status("attn_tc_kernel")) != cudaSuccess) return e;
  } else {
    // fp32 caches: CUDA-core kernel (fp32 products keep fp32 accuracy)
    const size_t smem = (size_t)(2 * kLeaf * kRowPad + kMaxG * kD) * sizeof(float);
    cudaFuncSetAttribute(attn_split_kernel<KT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int64_t grid = w.items_max < 148 * 3 ? w.items_max : 148 * 3;
    trace_begin(ZHA_TRACE_ATTN, c.stream);
    attn_split_kernel<KT><<<(unsigned)grid, 256, smem, c.stream>>>(aa);
    trace_end(ZHA_TRACE_ATTN, c.stream);
    count_launch();
    if ((e = launch_status("attn_split_kernel")) != cudaSuccess) return e;
  }

  // items of one unit: at most ceil((C1 + 2) / cps) + nr
  const int64_t items_unit = (w.C1 + 2 + w.cps - 1) / w.cps + w.nr;
  if (items_unit <= kCombBlock) {
    combine_warp_kernel<KT><<<(unsigned)w.units, kMaxG * 32, 0, c.stream>>>(ag, pair_off, aa.partials,
                                                                            (KT*)c.O, c.lse);
    count_launch();
    return launch_status("combine_warp_kernel");
  }
  const int64_t nbl = (items_unit + kCtaItems - 1) / kCtaItems;
  combine_cta_kernel<KT><<<(unsigned)(w.units * ag.G * nbl), 256, 0, c.stream>>>(ag, pair_off, aa.partials, nbl,
                                                                                 (KT*)c.O, c.lse);
  count_launch();
  if ((e = launch_status("combine_cta_kernel")) != cudaSuccess) return e;
  if (nbl > 1) {
    combine_cta_blocks_kernel<KT><<<(unsigned)w.units, kMaxG * 32, 0, c.stream>>>(ag, pair_off, aa.partials,
                                                                                  (KT*)c.O, c.lse);
    count_launch();
    return launch_status("combine_cta_blocks_kernel");
  }
  return cudaSuccess;
}

cudaError_t attention(const AttnCall& c) {
  return c.g->dtype == ZHA_BF16 ? attention_t<__nv_bfloat16>(c) : attention_t<float>(c);
}

}  // namespace zha
