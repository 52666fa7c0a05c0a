// Internal helpers shared by the ZHA kernels: geometry arithmetic, buffer layouts,
// exact number conversions, block reductions and the device status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "zha.h"

namespace zha {

constexpr int kD = 128;          // head dimension the kernels support
constexpr int kLeaf = 64;        // keys per leaf chunk
constexpr int kMaxR = 16;        // reference queries per KV head
constexpr int kMaxG = 8;         // query heads per KV head
constexpr int kMaxDepth = 8;
constexpr int kRange = 1024;     // chunk ids per union-building block
constexpr size_t kAlign = 256;
// Floats per split-KV partial: o[d], the running max m and sum l, padded so that every
// partial starts on a 16-byte boundary (vector stores).
constexpr int kPartStride = kD + 4;

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// geometry (host)
// ---------------------------------------------------------------------------

inline int64_t span_of(const zha_geom& g, int level) {
  int64_t s = g.leaf;
  for (int l = 1; l < level; ++l) s *= g.branch;
  return s;
}

inline int64_t ncap_of(const zha_geom& g, int level) { return g.t_cap / span_of(g, level); }

inline int elem_bytes(const zha_geom& g) { return g.dtype == ZHA_BF16 ? 2 : 4; }

// Bounds that keep every byte count and offset the library forms far inside 64-bit
// arithmetic (checked in double, which is exact at these magnitudes up to rounding that
// cannot cross the bound by more than one part in 2^52): one layer's cache, counted at
// 4 bytes per element, and the largest per-call array (8 bytes per query head per leaf
// chunk) each at most 2^48 bytes.
constexpr double kMaxBytes = 281474976710656.0;  // 2^48
inline bool cache_fits(const zha_geom& g) {
  return (double)g.B * g.Hkv * (double)g.t_cap * kD * 4.0 <= kMaxBytes;
}
inline bool call_fits(const zha_geom& g, int64_t nq) {
  return (double)g.B * (double)nq * g.Hq * (double)(g.t_cap / kLeaf + 2) * 8.0 <= kMaxBytes;
}

struct TreeLayout {
  zha_level_layout lv[kMaxDepth + 1];  // index = level (1..depth)
  size_t bytes;
};

inline TreeLayout tree_layout(const zha_geom& g) {
  TreeLayout t{};
  size_t off = 0;
  for (int l = 1; l <= g.depth; ++l) {
    zha_level_layout& L = t.lv[l];
    L.span = span_of(g, l);
    L.n_cap = g.t_cap / L.span;
    const size_t nodes = (size_t)g.B * g.Hkv * (size_t)L.n_cap;
    L.k_route_off = off;
    off = align_up(off + nodes * g.R * g.d * elem_bytes(g));
    L.b_hat_off = off;
    off = align_up(off + nodes * g.R * sizeof(float));
    L.F_off = off;
    off = align_up(off + nodes * g.R * sizeof(float));
    L.k_state_off = off;
    off = align_up(off + nodes * g.R * g.d * sizeof(float));
  }
  t.bytes = off;
  return t;
}

// Split size (chunks per attention work item) chosen from the geometry only, so that
// the workspace bound is known on the host: about 4K items per call (a few dozen per
// SM), >= 16 chunks each.
#ifndef ZHA_SPLIT_ITEMS
#define ZHA_SPLIT_ITEMS 4096                     // target number of attention work items
#endif
inline int64_t chunks_per_split(int64_t units, int64_t c1) {
  const int64_t total = units * (c1 + 2);
  int64_t cps = (total + ZHA_SPLIT_ITEMS - 1) / ZHA_SPLIT_ITEMS;
  return cps < 16 ? 16 : cps;
}

struct RouteWs {
  size_t cand_ids, cand_score, cand_mass, selA, selB, cand_cnt, selA_cnt, selB_cnt, pos, bytes;
  int64_t C1, C2;
};

inline RouteWs route_ws(const zha_geom& g, int nq, size_t base = 0) {
  RouteWs w{};
  const int64_t nqh = (int64_t)g.B * nq * g.Hq;
  w.C1 = ncap_of(g, 1);
  w.C2 = g.depth >= 2 ? ncap_of(g, 2) : 1;
  if (w.C2 < 1) w.C2 = 1;
  size_t off = base;
  w.cand_ids = off;   off = align_up(off + (size_t)nqh * w.C1 * 4);
  w.cand_score = off; off = align_up(off + (size_t)nqh * w.C1 * 8);
  w.cand_mass = off;  off = align_up(off + (size_t)nqh * w.C1 * 8);
  w.selA = off;       off = align_up(off + (size_t)nqh * w.C2 * 4);
  w.selB = off;       off = align_up(off + (size_t)nqh * w.C2 * 4);
  w.cand_cnt = off;   off = align_up(off + (size_t)nqh * 4);
  w.selA_cnt = off;   off = align_up(off + (size_t)nqh * 4);
  w.selB_cnt = off;   off = align_up(off + (size_t)nqh * 4);
  w.pos = off;        off = align_up(off + (size_t)g.B * nq * 8);
  w.bytes = off;
  return w;
}

struct AttnWs {
  size_t stage_ids, stage_mask, stage_cnt, pair_off, partials, pos, bytes;
  int64_t units, nr, pairs, cps, items_max, C1;
};

// cps = 0: the default split size; otherwise that many chunks per work item.
inline AttnWs attn_ws(const zha_geom& g, int nq, size_t base = 0, int64_t cps = 0) {
  AttnWs w{};
  const int G = g.Hq / g.Hkv;
  w.units = (int64_t)g.B * nq * g.Hkv;
  w.C1 = ncap_of(g, 1);
  w.nr = (w.C1 + 1 + kRange - 1) / kRange;
  w.pairs = w.units * w.nr;
  w.cps = cps > 0 ? cps : chunks_per_split(w.units, w.C1);
  w.items_max = w.pairs + (w.units * (w.C1 + 2) + w.cps - 1) / w.cps;
  size_t off = base;
  w.stage_ids = off;  off = align_up(off + (size_t)w.pairs * (kRange + 2) * 4);
  w.stage_mask = off; off = align_up(off + (size_t)w.pairs * (kRange + 2) * 4);
  w.stage_cnt = off;  off = align_up(off + (size_t)w.pairs * 4);
  w.pair_off = off;   off = align_up(off + (size_t)(w.pairs + 1) * 4);
  w.partials = off;   off = align_up(off + (size_t)w.items_max * G * kPartStride * 4);
  w.pos = off;        off = align_up(off + (size_t)g.B * nq * 8);
  w.bytes = off;
  return w;
}

// Query-tile attention for prefill (zha_prefill_attn): sub-tiles of Qt = kPrefillRows / G
// consecutive queries x the G heads of one KV head, two per tile; per (tile, range of
// kRange chunk ids) the union entries (chunk id, a 128-bit mask per sub-tile of the rows
// that selected it) and a count.
constexpr int kPrefillRows = 128;

struct PrefillWs {
  size_t ent_ids, ent_mask, ent_cnt, bytes;
  int Qt;
  int64_t nqt, tiles, nr;
};

PrefillWs prefill_ws(const zha_geom& g, int nq, size_t base = 0);

// Host-side launch counter (exported as zha_launch_count).
extern std::atomic<int64_t> g_launches;
inline void count_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// The error of the last failing CUDA call, kept for zha_last_error().
void note_cuda_error(cudaError_t e, const char* where);
inline cudaError_t launch_status(const char* kernel) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) note_cuda_error(e, kernel);
  return e;
}

// Event tracing around chosen kernels (zha_trace): record before / after one launch.
struct Tracer {
  void* const* start = nullptr;
  void* const* stop = nullptr;
  int n = 0, done = 0;
};
extern Tracer g_trace[5];
inline void trace_begin(int which, cudaStream_t s) {
  Tracer& t = g_trace[which];
  if (t.done < t.n) cudaEventRecord((cudaEvent_t)t.start[t.done], s);
}
inline void trace_end(int which, cudaStream_t s) {
  Tracer& t = g_trace[which];
  if (t.done < t.n) { cudaEventRecord((cudaEvent_t)t.stop[t.done], s); ++t.done; }
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void set_status(int32_t* st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

// bf16 -> fp64 exactly, with integer operations: a normal bf16 value maps to the double
// with the same sign, the exponent rebased from 127 to 1023, the 7 mantissa bits on top
// of the 52-bit mantissa.  Zero and subnormals take the (exact) float path.
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t h) {
  const uint32_t mag = h & 0x7fffu;
  if ((mag & 0x7f80u) == 0u || (mag & 0x7f80u) == 0x7f80u) {
    return (double)__uint_as_float(h << 16);
  }
  const uint32_t hi = ((h & 0x8000u) << 16) | ((mag + ((1023u - 127u) << 7)) << 13);
  return __hiloint2double((int)hi, 0);
}

__device__ __forceinline__ double to_f64(float x) { return (double)x; }
__device__ __forceinline__ double to_f64(__nv_bfloat16 x) {
  return bf16_bits_to_f64((uint32_t)__bfloat16_as_ushort(x));
}
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// Element i of a 16-byte vector of KT, without taking the vector's address (i is a
// compile-time constant after unrolling, so this folds to a register move or shift).
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int w) {
  return w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
}
template <typename KT> __device__ __forceinline__ float u4_elem(const uint4& v, int i);
template <> __device__ __forceinline__ float u4_elem<float>(const uint4& v, int i) {
  return __uint_as_float(u4_word(v, i));
}
template <> __device__ __forceinline__ float u4_elem<__nv_bfloat16>(const uint4& v, int i) {
  const uint32_t w = u4_word(v, i >> 1);
  return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

// fp64 -> storage type, a single round-to-nearest-even.
__device__ __forceinline__ __nv_bfloat16 f64_to_bf16_rn(double x) {
  unsigned short r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(x));
  return __ushort_as_bfloat16(r);
}
template <typename T> __device__ __forceinline__ T from_f64(double x);
template <> __device__ __forceinline__ float from_f64<float>(double x) { return __double2float_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f64<__nv_bfloat16>(double x) { return f64_to_bf16_rn(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ double shfl_xor_f64(double v, int m) { return __shfl_xor_sync(0xffffffffu, v, m); }

// D[8x8] += A[8x4] . B[4x8] in fp64 on the tensor cores (lane layout of mma.m8n8k4.f64:
// a = A[lane/4][lane%4], b = B[lane%4][lane/4], (d0, d1) = D[lane/4][2*(lane%4) + {0,1}]).
__device__ __forceinline__ void mma_f64(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d0), "+d"(d1) : "d"(a), "d"(b));
}

// First index i in [0, cnt) of an ascending list with lst[i] >= key (cnt if none), found by
// the whole warp with a 32-way search: every round probes 32 positions and keeps the
// segment where the list crosses key (about log32(cnt) dependent loads).  All lanes return
// the same index.
__device__ __forceinline__ int warp_lower_bound(const int* lst, int cnt, int64_t key) {
  const int lane = threadIdx.x & 31;
  int x0 = 0, x1 = cnt;                              // the answer lies in [x0, x1]
  while (x1 - x0 > 32) {
    const int step = (x1 - x0 + 31) / 32;
    const int idx = x0 + (lane + 1) * step - 1;
    const bool below = idx < x1 && lst[idx] < key;
    const int nx0 = x0 + __popc(__ballot_sync(0xffffffffu, below)) * step;
    x1 = nx0 + step < x1 ? nx0 + step : x1;
    x0 = nx0;
  }
  const bool below = x0 + lane < x1 && lst[x0 + lane] < key;
  return x0 + __popc(__ballot_sync(0xffffffffu, below));
}

// Position of the query of (b, qi): from q_pos, or the uniform position when q_pos is null.
__device__ __forceinline__ int64_t query_pos(const int64_t* q_pos, int64_t uniform, int64_t bq) {
  return q_pos ? q_pos[bq] : uniform;
}

// Visible full nodes of size `span` for a query at position t.
__device__ __forceinline__ int64_t visible_nodes(int64_t t, int64_t span) {
  return ((t / kLeaf) * kLeaf) / span;
}

// ---------------------------------------------------------------------------
// internal calls composed by the C ABI
// ---------------------------------------------------------------------------

struct RouteCall {
  const zha_geom* g;
  int nq;
  const void* Q;
  const int64_t* q_pos;          // [B, nq] device, or null: every query at pos_uniform
  int64_t pos_uniform;
  double p;
  void* tree;                    // tree buffer (route_all) or the K cache (flat_select)
  int* leaf_ids;
  int* leaf_cnt;
  int leaf_cap;
  int* level_cnt;
  int* level_ids;
  char* ws;                      // workspace base, layout route_ws(g, nq, 0)
  int32_t* dev_status;
  cudaStream_t stream;
  const double* p_levels = nullptr;  // host [depth]: level l selects with p_levels[l-1]; null: p
  const int32_t* k_levels = nullptr; // host [depth]: level l keeps its k_levels[l-1] best (top-K)
};

struct AttnCall {
  const zha_geom* g;
  int nq;
  const void* Q;
  const void* K;
  const void* V;
  const int64_t* q_pos;
  int64_t pos_uniform;
  int dense;                     // 1: every key [0, t] (baseline), 0: the routed index set
  const int* leaf_ids;
  const int* leaf_cnt;
  int leaf_cap;
  void* O;
  float* lse;
  char* ws;                      // workspace base, layout attn_ws(g, nq, 0, cps)
  int32_t* dev_status;
  cudaStream_t stream;
  int64_t cps = 0;               // chunks per work item; 0: the default of attn_ws
};

struct PrefillCall {
  const zha_geom* g;
  int nq;
  const void* Q;
  const void* K;
  const void* V;
  const int64_t* q_pos;
  const int* leaf_ids;
  const int* leaf_cnt;
  int leaf_cap;
  void* O;
  float* lse;
  char* ws;                      // workspace base, layout prefill_ws(g, nq, 0)
  int32_t* dev_status;
  cudaStream_t stream;
};

cudaError_t prefill_attention(const PrefillCall& c);
cudaError_t tree_extend(const zha_geom& g, const void* K, const float* qref, void* tree,
                        int64_t t_old, int64_t t_new, cudaStream_t s);
cudaError_t append_tokens(const zha_geom& g, void* K, void* V, const void* k_new,
                          const void* v_new, int64_t t_old, int n_new, cudaStream_t s);
cudaError_t route_all(const RouteCall& c);
cudaError_t flat_select(const RouteCall& c);
cudaError_t attention(const AttnCall& c);
// bf16 split-KV gather on tensor cores (zha_attn_tc.cu)
// Flat indexer scores of bf16 caches on the tensor cores: F_C(q) of every visible chunk of
// every query head, into the routing workspace's candidate arrays (ids, scores, counts).
cudaError_t flat_tc_launch(const zha_geom& g, int nq, const void* Q, const void* K, const int64_t* q_pos,
                          int64_t pos_uniform, int64_t C1, int* cand_ids, double* cand_score, int* cand_cnt,
                          int32_t* dev_status, cudaStream_t stream);
// Tensor maps and device facts shared by the TMA-fed kernels (zha_attn_tc.cu).
// make_kv_map: a [units, t_cap, 128] bf16 cache as a 3-D map of 64 x 64 boxes, 128B swizzle.
bool make_kv_map(CUtensorMap* map, const void* base, int64_t units, int64_t t_cap);
int sm_count();
// The bounded-wait check (zha_check_bounded_wait).
cudaError_t wait_check_launch(long long polls, int32_t* dev_status, long long* out, cudaStream_t stream);
cudaError_t attn_tc_launch(const AttnCall& c, const AttnWs& w, const int* stage_ids,
                           const unsigned int* stage_mask, const int* stage_cnt, const int* pair_off,
                           float* partials);

}  // namespace zha
