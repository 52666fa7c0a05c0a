// Split-KV gather attention for bf16 caches on sm_100a: TMA-fed, tensor-core scored.
//
// One persistent CTA per SM walks the work items (splits of the union-of-heads chunk
// lists built by union_kernel / plan_kernel).  A producer warp streams every selected
// 64-key block of K and V into a 4-stage shared-memory ring with 3-D TMA loads
// (cp.async.bulk.tensor, 128-byte swizzle, completion on mbarriers; no multicast).  Four
// consumer warps each own 16 keys of every block and run, for the G <= 8 query heads that
// share the block (GQA),
//     S^T[16 keys x 8 heads] = K_blk . Q^T          (mma.sync m16n8k16, bf16 in, fp32 acc)
//     online softmax per head (fp32, base 2), heads outside the block's mask at -inf
//     O^T[128 x 8]          += V_blk^T . P^T        (P rounded to bf16)
// and at the end of an item the four warps' (m, l, O) are merged into one split partial
// (arXiv 2610.42112 App. D-B1: d_v values and two softmax statistics per split).
// The kernel is bound by HBM bandwidth: every selected block of a KV group crosses HBM once.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "zha_internal.cuh"
#include "zha_ptx.cuh"

namespace zha {

namespace tc {

#ifndef ZHA_ATTN_STAGES
#define ZHA_ATTN_STAGES 4
#endif
constexpr int kStages = ZHA_ATTN_STAGES;         // 32 KiB each; 4..6 keep HBM saturated
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = 64 * 128;              // 64 rows x 64 bf16, one swizzled box
constexpr int kStageBytes = 4 * kBoxBytes;       // K lo/hi, V lo/hi
constexpr uint32_t kTxBytes = kStageBytes;
using namespace ptx;

struct Smem {
  unsigned char stage[kStages][kStageBytes];     // 1024-byte aligned (swizzle atoms)
  float o[kConsumerWarps][kMaxG][kD];            // per-warp O^T for the item merge
  float ml[kConsumerWarps][kMaxG][2];
  int2 meta[kStages];                            // (key count, head mask) of each stage
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  int abort;                                     // set once any wait of the CTA gave up
  int zero;                                      // always 0
};

struct Args {
  int B, nq, Hq, Hkv, G;
  int64_t t_cap;
  const int64_t* q_pos;
  int64_t pos_uniform;
  int64_t nr, cps;
  const __nv_bfloat16* Q;
  const int* stage_ids;
  const unsigned int* stage_mask;
  const int* stage_cnt;
  const int* pair_off;
  int64_t pairs;
  float* partials;
  int32_t* dev_status;
};

struct ItemInfo {
  int64_t pair, u, bq, unit_kv;   // unit_kv = b * Hkv + hk (tensor-map z coordinate)
  int hk, e0, e1;
  int64_t t, vstart, nvis;
};

__device__ __forceinline__ ItemInfo item_info(const Args& a, int64_t item) {
  ItemInfo it;
  int64_t lo = 0, hi = a.pairs;                  // last pair with pair_off[pair] <= item
  while (hi - lo > 1) { const int64_t m = (lo + hi) >> 1; if (a.pair_off[m] <= item) lo = m; else hi = m; }
  it.pair = lo;
  const int64_t sub = item - a.pair_off[lo];
  it.u = lo / a.nr;
  it.bq = it.u / a.Hkv;
  it.hk = (int)(it.u % a.Hkv);
  it.unit_kv = (it.bq / a.nq) * a.Hkv + it.hk;
  it.t = query_pos(a.q_pos, a.pos_uniform, it.bq);
  it.vstart = (it.t / kLeaf) * kLeaf;
  it.nvis = it.vstart / kLeaf;
  const int cnt = a.stage_cnt[lo];
  it.e0 = (int)(sub * a.cps);
  it.e1 = (int)((sub + 1) * a.cps < cnt ? (sub + 1) * a.cps : cnt);
  return it;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, Args a) {
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t total_items = a.pair_off[a.pairs];

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], kConsumerWarps); }
    sm.abort = 0;
    sm.zero = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one lane issues the TMA loads ----------------
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&kmap) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&vmap) : "memory");
      long long it_count = 0;
      long long issued[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        const ItemInfo info = item_info(a, item);
        const int* ids = a.stage_ids + info.pair * (kRange + 2);
        const unsigned int* msk = a.stage_mask + info.pair * (kRange + 2);
        for (int e = info.e0; e < info.e1; ++e, ++it_count) {
          const int s = (int)(it_count % kStages);
          if (it_count >= kStages) {
            if (!mbar_wait(&sm.empty[s], (uint32_t)(((it_count / kStages) - 1) & 1), &sm.abort)) {
              set_status(a.dev_status, ZHA_ERR_DEVICE);
              atomicExch(&sm.abort, 1);
              ok = false;
              break;
            }
          }
          if (*(volatile int*)&sm.abort) { ok = false; break; }
          const int id = ids[e];
          int k0, len;
          if (id < 0) { k0 = 0; len = 1; }
          else if (id == info.nvis) { k0 = (int)info.vstart; len = (int)(info.t - info.vstart + 1); }
          else { k0 = id * kLeaf; len = kLeaf; }
          sm.meta[s] = make_int2(len, (int)msk[e]);
          mbar_arrive_tx(&sm.full[s], kTxBytes);
          unsigned char* st = sm.stage[s];
          const int z = (int)info.unit_kv;
          tma_load_3d(st + 0 * kBoxBytes, &kmap, 0, k0, z, &sm.full[s]);
          tma_load_3d(st + 1 * kBoxBytes, &kmap, 64, k0, z, &sm.full[s]);
          tma_load_3d(st + 2 * kBoxBytes, &vmap, 0, k0, z, &sm.full[s]);
          tma_load_3d(st + 3 * kBoxBytes, &vmap, 64, k0, z, &sm.full[s]);
          ++issued[s];
        }
      }
      // drain: no TMA write may land after the CTA exits (the copies complete on their
      // own; this wait ignores `abort`)
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0 && !mbar_wait(&sm.full[s], (uint32_t)((issued[s] - 1) & 1), &sm.zero))
          set_status(a.dev_status, ZHA_ERR_DEVICE);
    }
    return;
  }

  // ---------------- consumers: 4 warps, warp w owns keys [16w, 16w + 16) ----------------
  const int g = lane >> 2, t4 = lane & 3;
  const float sl2 = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)
  long long it_count = 0;
  for (int64_t item = blockIdx.x; item < total_items; item += gridDim.x) {
    const ItemInfo info = item_info(a, item);
    // B fragments of Q^T: head g, dims 16kk + 2t4 (+1) and + 8 (heads >= G are zero)
    uint32_t qb[8][2];
    {
      const int h = g;
      const __nv_bfloat16* qrow = a.Q + ((info.bq * a.Hq) + info.hk * a.G + (h < a.G ? h : 0)) * kD;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        uint32_t w0 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t4);
        uint32_t w1 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t4 + 8);
        qb[kk][0] = h < a.G ? w0 : 0u;
        qb[kk][1] = h < a.G ? w1 : 0u;
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // heads 2t4, 2t4+1
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    for (int e = info.e0; e < info.e1; ++e, ++it_count) {
      const int s = (int)(it_count % kStages);
      if (!mbar_wait(&sm.full[s], (uint32_t)((it_count / kStages) & 1), &sm.abort)) {
        set_status(a.dev_status, ZHA_ERR_DEVICE);
        atomicExch(&sm.abort, 1);
        continue;      // every later wait of the CTA now fails at once; barriers stay aligned
      }
      const int2 meta = sm.meta[s];
      const uint32_t base = smem_u32(sm.stage[s]);
      // S^T = K . Q^T for keys 16w + [0, 16)
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int mi = lane >> 3, r8 = lane & 7;
        const int row = warp * 16 + r8 + ((mi & 1) << 3);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int box = kk >> 2;                       // dims 0-63 | 64-127
          const int chunk = ((kk & 3) << 1) + (mi >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(base + box * kBoxBytes + swz(row, chunk), a0, a1, a2, a3);
          mma_bf16(sc, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
        }
      }
      // mask: keys beyond the block's length, heads outside its mask
      const int key0 = warp * 16 + g, key1 = key0 + 8;
      const int hA = 2 * t4, hB = hA + 1;
      const bool hAok = (meta.y >> hA) & 1, hBok = (meta.y >> hB) & 1;
      float s00 = (key0 < meta.x && hAok) ? sc[0] * sl2 : -INFINITY;
      float s01 = (key0 < meta.x && hBok) ? sc[1] * sl2 : -INFINITY;
      float s10 = (key1 < meta.x && hAok) ? sc[2] * sl2 : -INFINITY;
      float s11 = (key1 < meta.x && hBok) ? sc[3] * sl2 : -INFINITY;
      float mxA = fmaxf(s00, s10), mxB = fmaxf(s01, s11);
#pragma unroll
      for (int x = 4; x < 32; x <<= 1) {
        mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, x));
        mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, x));
      }
      const float nA = fmaxf(m0, mxA), nB = fmaxf(m1, mxB);
      const float uA = nA == -INFINITY ? 0.f : nA, uB = nB == -INFINITY ? 0.f : nB;
      const float aA = exp2f(m0 - uA), aB = exp2f(m1 - uB);      // m = -inf -> 0
      const float p00 = exp2f(s00 - uA), p10 = exp2f(s10 - uA);
      const float p01 = exp2f(s01 - uB), p11 = exp2f(s11 - uB);
      float sA = p00 + p10, sB = p01 + p11;
#pragma unroll
      for (int x = 4; x < 32; x <<= 1) {
        sA += __shfl_xor_sync(0xffffffffu, sA, x);
        sB += __shfl_xor_sync(0xffffffffu, sB, x);
      }
      l0 = l0 * aA + sA;
      l1 = l1 * aB + sB;
      m0 = nA;
      m1 = nB;
#pragma unroll
      for (int i = 0; i < 8; ++i) { o[i][0] *= aA; o[i][1] *= aB; o[i][2] *= aA; o[i][3] *= aB; }
      // P^T (keys x heads) as the B fragment: lane needs head g, keys 2t4, 2t4+1 (+8)
      const uint32_t pk_lo = pack_bf16(p00, p01);      // key g,     heads 2t4, 2t4+1
      const uint32_t pk_hi = pack_bf16(p10, p11);      // key g + 8, heads 2t4, 2t4+1
      const int src0 = ((2 * t4) << 2) + (g >> 1), src1 = ((2 * t4 + 1) << 2) + (g >> 1);
      const uint32_t v0 = __shfl_sync(0xffffffffu, pk_lo, src0);
      const uint32_t v1 = __shfl_sync(0xffffffffu, pk_lo, src1);
      const uint32_t v2 = __shfl_sync(0xffffffffu, pk_hi, src0);
      const uint32_t v3 = __shfl_sync(0xffffffffu, pk_hi, src1);
      const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;
      const uint32_t pb0 = __byte_perm(v0, v1, sel);
      const uint32_t pb1 = __byte_perm(v2, v3, sel);
      // O^T += V^T . P^T for d = 16mt + [0, 16)
      {
        const int mi = lane >> 3, r8 = lane & 7;
        const int key = warp * 16 + r8 + ((mi >> 1) << 3);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int box = mt >> 2;
          const int chunk = ((mt & 3) << 1) + (mi & 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(base + 2 * kBoxBytes + box * kBoxBytes + swz(key, chunk), a0, a1, a2, a3);
          mma_bf16(o[mt], a0, a1, a2, a3, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    // merge the four warps' states into the item's partial; this lane holds O^T at
    // d = 16mt + g (+8) for heads 2t4 and 2t4 + 1
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      sm.o[warp][2 * t4][mt * 16 + g] = o[mt][0];
      sm.o[warp][2 * t4 + 1][mt * 16 + g] = o[mt][1];
      sm.o[warp][2 * t4][mt * 16 + g + 8] = o[mt][2];
      sm.o[warp][2 * t4 + 1][mt * 16 + g + 8] = o[mt][3];
    }
    if (g == 0) {
      sm.ml[warp][2 * t4][0] = m0; sm.ml[warp][2 * t4][1] = l0;
      sm.ml[warp][2 * t4 + 1][0] = m1; sm.ml[warp][2 * t4 + 1][1] = l1;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    {
      const int d = threadIdx.x;                       // 0..127
      for (int h = 0; h < a.G; ++h) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.ml[w][h][0]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float f = exp2f(sm.ml[w][h][0] - M);
            L = fmaf(f, sm.ml[w][h][1], L);
            acc = fmaf(f, sm.o[w][h][d], acc);
          }
        }
        float* P = a.partials + ((int64_t)item * a.G + h) * kPartStride;
        P[d] = acc;
        if (d == 0) { P[kD] = M; P[kD + 1] = L; }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Flat indexer scores (the exact-chunk-score baseline) on the same TMA ring: every
// visible 64-key chunk of a KV group streams through shared memory once; consumer warp w
// takes the chunks w, w + 4, ... of the CTA's sequence (ring stage s always belongs to warp
// s % 4), computes S^T[64 keys x 8 heads] = K_chunk . Q^T with mma.sync bf16 (fp32
// accumulate) and reduces it to F_C(q) = max + log(sum exp(s - max)) per head.
// ---------------------------------------------------------------------------

constexpr int kFlatStages = 8;                   // a multiple of the consumer warps
constexpr int kFlatChunksPerItem = 64;
constexpr uint32_t kFlatTxBytes = 2 * kBoxBytes;

struct FlatSmem {
  unsigned char stage[kFlatStages][2 * kBoxBytes];   // K dims 0-63 | 64-127 of one chunk
  unsigned long long full[kFlatStages];
  unsigned long long empty[kFlatStages];
  int abort;
  int zero;
};

struct FlatTcArgs {
  int B, nq, Hq, Hkv, G;
  int64_t t_cap;
  const int64_t* q_pos;
  int64_t pos_uniform;
  const __nv_bfloat16* Q;
  int64_t C1, nblk;                              // chunk blocks (of kFlatChunksPerItem) per unit
  int* cand_ids;
  double* cand_score;
  int* cand_cnt;
  int32_t* dev_status;
};

struct FlatItem {
  int64_t bq, unit_kv, blk, nvis;
  int hk, c0, c1;
};

__device__ __forceinline__ FlatItem flat_item(const FlatTcArgs& a, int64_t item) {
  FlatItem f;
  const int64_t u = item / a.nblk;
  f.blk = item % a.nblk;
  f.bq = u / a.Hkv;
  f.hk = (int)(u % a.Hkv);
  f.unit_kv = (f.bq / a.nq) * a.Hkv + f.hk;
  const int64_t t = query_pos(a.q_pos, a.pos_uniform, f.bq);
  f.nvis = (t >= 0 && t < a.t_cap) ? visible_nodes(t, kLeaf) : 0;
  const int64_t lo = f.blk * kFlatChunksPerItem;
  f.c0 = (int)(lo < f.nvis ? lo : f.nvis);
  f.c1 = (int)(lo + kFlatChunksPerItem < f.nvis ? lo + kFlatChunksPerItem : f.nvis);
  return f;
}

__global__ void __launch_bounds__(kThreads, 1)
flat_tc_kernel(const __grid_constant__ CUtensorMap kmap, FlatTcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  FlatSmem& sm = *reinterpret_cast<FlatSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t total_items = (int64_t)a.B * a.nq * a.Hkv * a.nblk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFlatStages; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], 1); }
    sm.abort = 0;
    sm.zero = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer: one lane issues the TMA loads ----------------
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)&kmap) : "memory");
      long long it_count = 0;
      long long issued[kFlatStages];
      for (int s = 0; s < kFlatStages; ++s) issued[s] = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        const FlatItem f = flat_item(a, item);
        for (int c = f.c0; c < f.c1; ++c, ++it_count) {
          const int s = (int)(it_count % kFlatStages);
          if (it_count >= kFlatStages) {
            if (!mbar_wait(&sm.empty[s], (uint32_t)(((it_count / kFlatStages) - 1) & 1), &sm.abort)) {
              set_status(a.dev_status, ZHA_ERR_DEVICE);
              atomicExch(&sm.abort, 1);
              ok = false;
              break;
            }
          }
          if (*(volatile int*)&sm.abort) { ok = false; break; }
          mbar_arrive_tx(&sm.full[s], kFlatTxBytes);
          tma_load_3d(sm.stage[s], &kmap, 0, c * kLeaf, (int)f.unit_kv, &sm.full[s]);
          tma_load_3d(sm.stage[s] + kBoxBytes, &kmap, 64, c * kLeaf, (int)f.unit_kv, &sm.full[s]);
          ++issued[s];
        }
      }
      // drain: no TMA write may land after the CTA exits
      for (int s = 0; s < kFlatStages; ++s)
        if (issued[s] > 0 && !mbar_wait(&sm.full[s], (uint32_t)((issued[s] - 1) & 1), &sm.zero))
          set_status(a.dev_status, ZHA_ERR_DEVICE);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, t4 = lane & 3;
  const float scale = 1.0f / sqrtf((float)kD);
  long long it_count = 0;
  for (int64_t item = blockIdx.x; item < total_items; item += gridDim.x) {
    const FlatItem f = flat_item(a, item);
    const int64_t qh0 = f.bq * a.Hq + (int64_t)f.hk * a.G;
    if (f.blk == 0 && warp == 0 && lane < a.G) a.cand_cnt[qh0 + lane] = (int)f.nvis;
    if (f.c0 >= f.c1) continue;
    uint32_t qb[8][2];
    {
      const __nv_bfloat16* qrow = a.Q + (qh0 + (g < a.G ? g : 0)) * kD;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t4);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t4 + 8);
        qb[kk][0] = g < a.G ? w0 : 0u;
        qb[kk][1] = g < a.G ? w1 : 0u;
      }
    }
    for (int c = f.c0; c < f.c1; ++c, ++it_count) {
      if ((int)(it_count % kConsumerWarps) != warp) continue;
      const int s = (int)(it_count % kFlatStages);
      if (!mbar_wait(&sm.full[s], (uint32_t)((it_count / kFlatStages) & 1), &sm.abort)) {
        set_status(a.dev_status, ZHA_ERR_DEVICE);
        atomicExch(&sm.abort, 1);
        continue;
      }
      const uint32_t base = smem_u32(sm.stage[s]);
      float sc[4][4];
      const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
        const int row = 16 * j + r8 + ((mi & 1) << 3);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int box = kk >> 2;
          const int chunk = ((kk & 3) << 1) + (mi >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(base + box * kBoxBytes + swz(row, chunk), a0, a1, a2, a3);
          mma_bf16(sc[j], a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      // lane holds keys 16j + g (+8) for heads 2t4 (values 0, 2) and 2t4 + 1 (values 1, 3)
      float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mA = fmaxf(mA, fmaxf(sc[j][0] * scale, sc[j][2] * scale));
        mB = fmaxf(mB, fmaxf(sc[j][1] * scale, sc[j][3] * scale));
      }
#pragma unroll
      for (int x = 4; x < 32; x <<= 1) {
        mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, x));
        mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, x));
      }
      float zA = 0.f, zB = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        zA += expf(sc[j][0] * scale - mA) + expf(sc[j][2] * scale - mA);
        zB += expf(sc[j][1] * scale - mB) + expf(sc[j][3] * scale - mB);
      }
#pragma unroll
      for (int x = 4; x < 32; x <<= 1) {
        zA += __shfl_xor_sync(0xffffffffu, zA, x);
        zB += __shfl_xor_sync(0xffffffffu, zB, x);
      }
      if (g == 0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int h = 2 * t4 + q;
          if (h < a.G) {
            double F = (double)(q ? mB : mA) + log((double)(q ? zB : zA));
            if (F == 0.0) F = 0.0;
            a.cand_ids[(qh0 + h) * a.C1 + c] = c;
            a.cand_score[(qh0 + h) * a.C1 + c] = F;
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Check of the bounded waits: warp 0 waits on an mbarrier that nothing ever completes, with
// the rings' own wait and `polls` as its limit; when it gives up it reports ZHA_ERR_DEVICE
// and raises `abort` as the ring kernels do.  Warp 1 waits on a second such barrier with a
// limit 64 times larger; it stops early, through `abort`, once warp 0 has given up.
// out[0], out[1] = the clock cycles each warp spent waiting, out[2] = 1 if warp 0 gave
// up, out[3] = 1 if warp 1 returned without its barrier completing.  No copy is in flight
// and nothing faults: the kernel ends normally.
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(64) wait_check_kernel(long long polls, int32_t* st, long long* out) {
  __shared__ unsigned long long bar[2];
  __shared__ int abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (lane != 0) return;
  const long long t0 = clock64();
  const bool ok = mbar_wait(&bar[warp], 0u, &abort, warp == 0 ? polls : polls * 64);
  const long long dt = clock64() - t0;
  if (!ok && warp == 0) {
    set_status(st, ZHA_ERR_DEVICE);
    atomicExch(&abort, 1);
  }
  out[warp] = dt;
  out[2 + warp] = ok ? 0 : 1;
}

}  // namespace tc

cudaError_t wait_check_launch(long long polls, int32_t* dev_status, long long* out, cudaStream_t stream) {
  tc::wait_check_kernel<<<1, 64, 0, stream>>>(polls, dev_status, out);
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [units, t_cap, 128] bf16 cache as a 3-D tensor map with 64 x 64 boxes, 128B swizzle.
bool make_kv_map(CUtensorMap* map, const void* base, int64_t units, int64_t t_cap) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)t_cap, (cuuint64_t)units};
  const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)t_cap * kD * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

cudaError_t attn_tc_launch(const AttnCall& c, const AttnWs& w, const int* stage_ids,
                           const unsigned int* stage_mask, const int* stage_cnt, const int* pair_off,
                           float* partials) {
  const zha_geom& g = *c.g;
  CUtensorMap km, vm;
  const int64_t units_kv = (int64_t)g.B * g.Hkv;
  if (!make_kv_map(&km, c.K, units_kv, g.t_cap) || !make_kv_map(&vm, c.V, units_kv, g.t_cap)) {
    note_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
    return cudaErrorInvalidValue;
  }
  tc::Args a{};
  a.B = g.B; a.nq = c.nq; a.Hq = g.Hq; a.Hkv = g.Hkv; a.G = g.Hq / g.Hkv; a.t_cap = g.t_cap;
  a.q_pos = c.q_pos; a.pos_uniform = c.pos_uniform; a.nr = w.nr; a.cps = w.cps;
  a.Q = (const __nv_bfloat16*)c.Q;
  a.stage_ids = stage_ids; a.stage_mask = stage_mask; a.stage_cnt = stage_cnt; a.pair_off = pair_off;
  a.pairs = w.pairs; a.partials = partials; a.dev_status = c.dev_status;
  const size_t smem = sizeof(tc::Smem) + 1024;
  cudaFuncSetAttribute(tc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int64_t grid = w.items_max < sm_count() ? w.items_max : sm_count();
  tc::attn_tc_kernel<<<(unsigned)grid, tc::kThreads, smem, c.stream>>>(km, vm, a);
  return cudaSuccess;
}

cudaError_t flat_tc_launch(const zha_geom& g, int nq, const void* Q, const void* K, const int64_t* q_pos,
                          int64_t pos_uniform, int64_t C1, int* cand_ids, double* cand_score, int* cand_cnt,
                          int32_t* dev_status, cudaStream_t stream) {
  CUtensorMap km;
  if (!make_kv_map(&km, K, (int64_t)g.B * g.Hkv, g.t_cap)) {
    note_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
    return cudaErrorInvalidValue;
  }
  tc::FlatTcArgs a{};
  a.B = g.B; a.nq = nq; a.Hq = g.Hq; a.Hkv = g.Hkv; a.G = g.Hq / g.Hkv; a.t_cap = g.t_cap;
  a.q_pos = q_pos; a.pos_uniform = pos_uniform;
  a.Q = (const __nv_bfloat16*)Q;
  a.C1 = C1;
  a.nblk = (C1 + tc::kFlatChunksPerItem - 1) / tc::kFlatChunksPerItem;
  if (a.nblk < 1) a.nblk = 1;
  a.cand_ids = cand_ids; a.cand_score = cand_score; a.cand_cnt = cand_cnt; a.dev_status = dev_status;
  const size_t smem = sizeof(tc::FlatSmem) + 1024;
  cudaFuncSetAttribute(tc::flat_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int64_t items = (int64_t)g.B * nq * g.Hkv * a.nblk;
  const int64_t grid = items < sm_count() ? items : sm_count();
  tc::flat_tc_kernel<<<(unsigned)(grid < 1 ? 1 : grid), tc::kThreads, smem, stream>>>(km, a);
  return cudaSuccess;
}

}  // namespace zha
