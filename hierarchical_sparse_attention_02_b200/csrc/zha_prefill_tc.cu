// Query-tile sparse attention for chunked prefill on the 5th-generation tensor cores.
//
// arXiv 2610.42112, App. A-B (Table I) counts the KV footprint of a tile of Q consecutive
// queries as the union of the leaf lists of its Q queries x G heads, while every query
// keeps its own output o(q) = Attn(q, K_I(q), V_I(q)) ("ZHA summary" page, Routing):
//   I(q) = {0} u (keys of the chunks in S_1(q)) u C_cur(q),   C_cur(q) = [V(t), t].
// Here a sub-tile is Qt = floor(128 / G) consecutive queries of one sequence and the G
// query heads of one KV head: M = Qt * G <= 128 rows (row r = query r / G, head r % G), the
// M of one tcgen05 MMA.  A CTA takes two consecutive sub-tiles at a time (a tile of 2 Qt
// queries): both share every K / V chunk load and run their softmax on separate warps, so
// the MMAs of one overlap the softmax of the other.  For every 64-key chunk of the tile's
// union the kernel computes, for each sub-tile,
//     S[128 x 64]  = Q_tile . K_chunk^T     (tcgen05.mma kind::f16, bf16 in, fp32 in TMEM)
//     P            = exp2(S * log2(e)/sqrt(d) - m)  per row, masked to the row's own keys
//     O[128 x 128] += P . V_chunk           (tcgen05.mma, P from TMEM, O in TMEM)
// with an online softmax per row whose running maximum is raised lazily (O in TMEM is
// rescaled only when a row's maximum grows by more than 2^8).  A row sees key j of chunk c
// iff c is in its S_1, or j = 0, or c is its own chunk and j <= t.
//
// Roles in one CTA of 576 threads, one tile after another (a persistent grid):
//   warps 0-15 softmax and epilogue: warp w serves sub-tile w / 8, the keys [32 h, 32 h + 32)
//              of each chunk and the output dims [64 h, 64 h + 64) for h = (w / 4) % 2, and
//              the rows 32 (w % 4) + lane (= its TMEM lanes); the two threads of a row share
//              their maxima through shared memory and an mbarrier (sub-tile u owns TMEM
//              columns [256 u, 256 u + 256)); each thread writes its 32 weights of P as
//              bf16 pairs over the first 16 of the 32 S columns it has just read, where the
//              P . V MMA reads them as its A operand;
//   warp 16    producer: TMA loads of the Q sub-tiles (4-D map) and of each chunk's K and V
//              (3-D maps, 128-byte swizzle) into a 4-stage ring; this GPU's memory only,
//              no multicast;
//   warp 17    TMEM allocation; lane 0 issues the MMAs and their commits.
// Every wait is bounded; a wait that gives up reports ZHA_ERR_DEVICE, the CTA stops, waits
// (bounded) for its copies and MMAs in flight, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "zha_internal.cuh"
#include "zha_ptx.cuh"

namespace zha {

namespace qt {

using namespace ptx;

constexpr int kRows = 128;                       // MMA M: rows of a sub-tile
constexpr int kSub = 2;                          // sub-tiles per tile
constexpr int kStages = 4;                       // K/V ring depth
constexpr int kBox = 64 * 128;                   // 64 rows x 128 bytes
constexpr int kKVBytes = 4 * kBox;               // K dims 0-63 | 64-127, V dims 0-63 | 64-127
constexpr int kQHalf = kRows * 128;              // 128 rows x 64 dims of Q
constexpr uint32_t kTmemCols = 512;              // per sub-tile: S0, S1 (64 each, P over them), O (128)
constexpr uint32_t kSubCols = 256;
constexpr uint32_t kColO = 128;
constexpr int kHalves = 2;                      // softmax threads per row (32 of its 64 keys each)
constexpr int kSoftWarps = 4 * kHalves * kSub;
constexpr int kProducerWarp = kSoftWarps, kMmaWarp = kSoftWarps + 1;
constexpr int kThreads = (kSoftWarps + 2) * 32;
constexpr float kLazy = 8.0f;                    // rescale O when a row max grows by > 2^8
constexpr uint32_t kIdescS = idesc_bf16(128, 64, 0);   // S = Q . K^T, both K-major
constexpr uint32_t kIdescPV = idesc_bf16(128, 128, 1); // O += P . V, V MN-major

struct alignas(1024) Smem {
  unsigned char q[kSub][2][kQHalf];              // per sub-tile two 128B-swizzled boxes [128 rows][64 dims]
  unsigned char kv[kStages][kKVBytes];
  uint4 meta_mask[kStages][kSub];                // rows of each sub-tile that selected the chunk
  int meta_id[kStages];                          // chunk id of each stage
  unsigned long long full[kStages], empty[kStages];
  unsigned long long q_full, q_empty;
  unsigned long long s_full[kSub][2], p_full[kSub][2], pv_done[kSub][2];
  unsigned long long o_free[kSub], drain;
  unsigned long long pair[kSub][4];              // the two warps (halves) of each row group
  float xmax[2][kSub][kHalves][kRows];           // row maxima (per entry) and sums (epilogue) of the
                                                 // two halves of a row, by entry parity
  uint32_t tmem_base;
  int abort, zero;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of the prefill kernel");

struct Args {
  int B, nq, Hq, Hkv, G, Qt, nqt;                // nqt: tiles of 2 Qt queries per KV unit
  int64_t t_cap, nr, tiles;
  const int64_t* q_pos;
  const int* ent_ids;                            // [tiles, nr, kRange]
  const uint4* ent_mask;                         // [tiles, nr, kRange, kSub] 128-bit row masks
  const int* ent_cnt;                            // [tiles, nr]
  __nv_bfloat16* O;
  float* lse;
  int32_t* dev_status;
};

struct Tile {
  int b, hk, q0;
  int64_t unit;                                  // b * Hkv + hk (K/V map z coordinate)
};

__device__ __forceinline__ Tile tile_of(const Args& a, int64_t tile) {
  Tile t;
  t.unit = tile / a.nqt;                          // tiles of one KV unit are consecutive
  t.q0 = (int)(tile % a.nqt) * kSub * a.Qt;
  t.b = (int)(t.unit / a.Hkv);
  t.hk = (int)(t.unit % a.Hkv);
  return t;
}

__device__ __forceinline__ int tile_entries(const Args& a, int64_t tile) {
  int n = 0;
  for (int64_t r = 0; r < a.nr; ++r) n += a.ent_cnt[tile * a.nr + r];
  return n;
}

// Up to 32 consecutive entries of one range of a tile, one per lane (nb = how many).
struct Batch {
  int c, nb;
  uint4 m0, m1;
};

// Walks a tile's entries in batches of at most 32 within one range.
struct BatchWalk {
  int64_t base, r, e0, cnt;
  __device__ void start(const Args& a, int64_t tile) {
    base = tile * a.nr;
    r = 0;
    e0 = 0;
    cnt = a.ent_cnt[base];
    while (cnt == 0 && r + 1 < a.nr) { ++r; cnt = a.ent_cnt[base + r]; }
  }
  // the next batch (nb = 0 once the tile's entries are exhausted); every lane calls it
  __device__ Batch load(const Args& a, int lane) {
    Batch b;
    b.nb = e0 < cnt ? (int)(cnt - e0 < 32 ? cnt - e0 : 32) : 0;
    b.c = 0;
    b.m0 = b.m1 = make_uint4(0u, 0u, 0u, 0u);
    if (lane < b.nb) {
      const int64_t slot = (base + r) * kRange + e0 + lane;
      b.c = a.ent_ids[slot];
      b.m0 = a.ent_mask[slot * kSub];
      b.m1 = a.ent_mask[slot * kSub + 1];
    }
    if (b.nb > 0) {
      e0 += 32;
      if (e0 >= cnt) {
        e0 = 0;
        do { ++r; cnt = r < a.nr ? a.ent_cnt[base + r] : 0; } while (cnt == 0 && r + 1 < a.nr);
      }
    }
    return b;
  }
};
static_assert(kSub == 2, "a batch carries the row masks of two sub-tiles");

__device__ __forceinline__ bool warp_wait(unsigned long long* b, uint32_t parity, int* abort) {
  const bool ok = __all_sync(0xffffffffu, mbar_wait_sleep(b, parity, abort));
  return ok;
}

__device__ __forceinline__ void give_up(Smem& sm, int32_t* st) {
  set_status(st, ZHA_ERR_DEVICE);
  atomicExch(&sm.abort, 1);
}

// 2^x on the SFU (approximate, flushes subnormal results to zero; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap, Args a) {
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], 1); }
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int u = 0; u < kSub; ++u) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&sm.s_full[u][i], 1);
        mbar_init(&sm.p_full[u][i], 4 * kHalves);
        mbar_init(&sm.pv_done[u][i], 1);
      }
      mbar_init(&sm.o_free[u], 4 * kHalves);
      for (int g4 = 0; g4 < 4; ++g4) mbar_init(&sm.pair[u][g4], kHalves);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    sm.zero = 0;
    mbar_init_fence();
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ producer
    // The whole warp reads the entries' chunk ids and row masks 32 at a time (one coalesced
    // load per lane, the next batch in flight while this one is issued); lane 0 waits for
    // the ring slots and issues the TMA copies.
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
    const uint32_t q_tx = (uint32_t)(kSub * 2 * 128 * a.G * a.Qt);
    long long it = 0, nq_loads = 0;
    long long issued[kStages] = {};
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < a.tiles && ok; tile += gridDim.x) {
      const Tile t = tile_of(a, tile);
      int okw = 1;
      if (lane == 0) {
        if (nq_loads > 0 && !mbar_wait_sleep(&sm.q_empty, (uint32_t)((nq_loads - 1) & 1), &sm.abort)) {
          okw = 0;
        } else {
          mbar_arrive_tx(&sm.q_full, q_tx);
          for (int u = 0; u < kSub; ++u) {         // a sub-tile past nq reads the fill value (0)
            tma_load_4d(sm.q[u][0], &qmap, 0, t.hk * a.G, t.q0 + u * a.Qt, t.b, &sm.q_full);
            tma_load_4d(sm.q[u][1], &qmap, 64, t.hk * a.G, t.q0 + u * a.Qt, t.b, &sm.q_full);
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
      ++nq_loads;
      BatchWalk w;
      w.start(a, tile);
      Batch cur = w.load(a, lane), nxt = w.load(a, lane);
      while (cur.nb > 0 && ok) {
        for (int k = 0; k < cur.nb; ++k, ++it) {
          const int s = (int)(it % kStages);
          okw = 1;
          if (lane == 0 && it >= kStages &&
              !mbar_wait_sleep(&sm.empty[s], (uint32_t)(((it / kStages) - 1) & 1), &sm.abort))
            okw = 0;
          if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
          if (lane == k) {                         // the entry's owner lane publishes its metadata
            sm.meta_id[s] = cur.c;
            sm.meta_mask[s][0] = cur.m0;
            sm.meta_mask[s][1] = cur.m1;
          }
          const int c = __shfl_sync(0xffffffffu, cur.c, k);
          __syncwarp();                            // the metadata is written before the arrival
          if (lane == 0) {
            mbar_arrive_tx(&sm.full[s], (uint32_t)kKVBytes);
            unsigned char* st = sm.kv[s];
            const int z = (int)t.unit;
            tma_load_3d(st + 0 * kBox, &kmap, 0, c * kLeaf, z, &sm.full[s]);
            tma_load_3d(st + 1 * kBox, &kmap, 64, c * kLeaf, z, &sm.full[s]);
            tma_load_3d(st + 2 * kBox, &vmap, 0, c * kLeaf, z, &sm.full[s]);
            tma_load_3d(st + 3 * kBox, &vmap, 64, c * kLeaf, z, &sm.full[s]);
            ++issued[s];
          }
        }
        cur = nxt;
        nxt = w.load(a, lane);
      }
    }
    if (lane == 0) {
      if (!ok) give_up(sm, a.dev_status);
      // drain: no copy may land after the CTA exits (bounded, independent of `abort`)
      for (int s = 0; s < kStages; ++s)
        if (issued[s] > 0 && !mbar_wait(&sm.full[s], (uint32_t)((issued[s] - 1) & 1), &sm.zero))
          set_status(a.dev_status, ZHA_ERR_DEVICE);
      if (nq_loads > 0 && !mbar_wait(&sm.q_full, (uint32_t)((nq_loads - 1) & 1), &sm.zero))
        set_status(a.dev_status, ZHA_ERR_DEVICE);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long j = 0, tl = 0;                   // entries and tiles of this CTA so far
      bool ok = true;
      // S of entry e overwrites the columns that held S and then P of entry e - 2: it waits
      // until the P . V MMA of e - 2 (issued after its P was written) has completed
      auto issue_s = [&](int u, long long e) -> bool {
        if (e >= 2 && !mbar_wait_sleep(&sm.pv_done[u][e & 1], (uint32_t)(((e >> 1) - 1) & 1), &sm.abort)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(sm.q[u][0]);
        const uint32_t ka = smem_u32(sm.kv[e % kStages]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16(tmem + u * kSubCols + (uint32_t)(e & 1) * 64,
                    sw128_desc(qa + (kk >> 2) * kQHalf + (kk & 3) * 32, 16, 1024),
                    sw128_desc(ka + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024), kIdescS, kk > 0 ? 1u : 0u);
        umma_commit(&sm.s_full[u][e & 1]);
        return true;
      };
      auto issue_pv = [&](int u, long long e, bool first_of_tile) -> bool {
        if (!mbar_wait_sleep(&sm.p_full[u][e & 1], (uint32_t)((e >> 1) & 1), &sm.abort)) return false;
        if (first_of_tile && tl > 0 && !mbar_wait_sleep(&sm.o_free[u], (uint32_t)((tl - 1) & 1), &sm.abort)) return false;
        tc_fence_after();
        // P of keys [16 kk, 16 kk + 16): columns 8 (kk % 2) of the S half 32 (kk / 2)
        const uint32_t pa = tmem + u * kSubCols + (uint32_t)(e & 1) * 64;
        const uint32_t va = smem_u32(sm.kv[e % kStages] + 2 * kBox);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ts(tmem + u * kSubCols + kColO, pa + (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8),
                       sw128_desc(va + kk * 2048, kBox, 1024), kIdescPV, (first_of_tile && kk == 0) ? 0u : 1u);
        umma_commit(&sm.pv_done[u][e & 1]);
        return true;
      };
      for (int64_t tile = blockIdx.x; tile < a.tiles && ok; tile += gridDim.x, ++tl) {
        const int n = tile_entries(a, tile);
        if (!mbar_wait_sleep(&sm.q_full, (uint32_t)(tl & 1), &sm.abort)) { ok = false; break; }
        tc_fence_after();
        for (int i = 0; i < n; ++i, ++j) {
          const int s = (int)(j % kStages);
          if (!mbar_wait_sleep(&sm.full[s], (uint32_t)((j / kStages) & 1), &sm.abort)) { ok = false; break; }
          if (!issue_s(0, j) || !issue_s(1, j)) { ok = false; break; }
          if (i >= 1) {
            if (!issue_pv(0, j - 1, i == 1) || !issue_pv(1, j - 1, i == 1)) { ok = false; break; }
            umma_commit(&sm.empty[(j - 1) % kStages]);
          }
        }
        if (!ok) break;
        if (n >= 1) {
          if (!issue_pv(0, j - 1, n == 1) || !issue_pv(1, j - 1, n == 1)) { ok = false; break; }
          umma_commit(&sm.empty[(j - 1) % kStages]);
        }
        umma_commit(&sm.q_empty);                  // Q is free once this tile's MMAs are done
      }
      if (!ok) give_up(sm, a.dev_status);
      // drain: every MMA this thread issued has completed before TMEM is freed
      umma_commit(&sm.drain);
      if (!mbar_wait(&sm.drain, 0u, &sm.zero)) set_status(a.dev_status, ZHA_ERR_DEVICE);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int u = warp >> 3;                     // sub-tile of this warp
    const int hf = (warp >> 2) & 1;              // half of the row: keys 32 hf.., dims 64 hf..
    const int r = (warp & 3) * 32 + lane;        // row = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + u * kSubCols;
    const uint32_t s_col = (uint32_t)hf * 32, o_col = kColO + (uint32_t)hf * 64;
    long long npair = 0;                         // phases of this row group's pair barrier
    const float sl2 = 1.4426950408889634f * 0.08838834764831845f;   // log2(e) / sqrt(128)
    long long j = 0, tl = 0;
    bool ok = true;
    // the two warps of this row group meet (bounded): shared-memory writes before it are seen
    // after it
    auto pair_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pair[u][warp & 3]);
      const bool k2 = warp_wait(&sm.pair[u][warp & 3], (uint32_t)(npair & 1), &sm.abort);
      ++npair;
      return k2;
    };
    for (int64_t tile = blockIdx.x; tile < a.tiles && ok; tile += gridDim.x, ++tl) {
      const Tile t = tile_of(a, tile);
      const int n = tile_entries(a, tile);
      // this row's query
      const int qi = t.q0 + u * a.Qt + r / a.G;
      const int h = t.hk * a.G + r % a.G;
      bool valid = r < a.Qt * a.G && qi < a.nq;
      int64_t pos = 0;
      if (valid) {
        pos = a.q_pos[(int64_t)t.b * a.nq + qi];
        if (pos < 0 || pos >= a.t_cap) valid = false;   // reported by the union kernel
      }
      const int64_t cur = valid ? pos / kLeaf : -1;    // the row's own chunk = n_vis(t)
      const uint32_t mword = (uint32_t)(r >> 5), mbit = 1u << (r & 31);
      float m = -INFINITY, l = 0.f;
      for (int i = 0; i < n; ++i, ++j) {
        const int s = (int)(j % kStages);
        if (!warp_wait(&sm.full[s], (uint32_t)((j / kStages) & 1), &sm.abort)) { ok = false; break; }
        const int c = sm.meta_id[s];
        const uint4 mk = sm.meta_mask[s][u];
        if (!warp_wait(&sm.s_full[u][j & 1], (uint32_t)((j >> 1) & 1), &sm.abort)) { ok = false; break; }
        tc_fence_after();
        float x[32];
        tmem_ld32(lane_addr + (uint32_t)(j & 1) * 64 + s_col, x);
        tmem_wait_ld();
        // visibility of the chunk's keys for this row: all of them (a selected chunk), the
        // keys up to t (its own chunk), key 0 (chunk 0), or none; this thread holds keys
        // 32 hf + k
        const uint32_t wsel = mword == 0 ? mk.x : mword == 1 ? mk.y : mword == 2 ? mk.z : mk.w;
        const bool sel = valid && (wsel & mbit) && c < cur;
        const bool own = valid && c == cur;
        const int lim = (sel ? 63 : (own ? (int)(pos - (int64_t)c * kLeaf) : (valid && c == 0 ? 0 : -1))) - 32 * hf;
        // A row sees all 32 of this thread's keys (lim >= 31) or none of them (lim < 0) on
        // every entry but its own chunk and chunk 0; only those few entries mask key by key.
        if (__any_sync(0xffffffffu, lim >= 0 && lim < 31)) {
#pragma unroll
          for (int k = 0; k < 32; ++k) x[k] = k <= lim ? x[k] : -INFINITY;
        }
        float mx;
        {
          float m4[4];                                 // independent chains of 3-input maxima
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const float* y = x + 8 * c4;
            m4[c4] = fmax3(fmax3(y[0], y[1], y[2]), fmax3(y[3], y[4], y[5]), fmaxf(y[6], y[7]));
          }
          mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * sl2;   // log2 units (-inf stays)
          if (lim < 0) mx = -INFINITY;               // the row sees none of these keys
        }
        // the row maximum over both halves
        sm.xmax[j & 1][u][hf][r] = mx;
        if (!pair_sync()) { ok = false; break; }
        mx = fmaxf(mx, sm.xmax[j & 1][u][hf ^ 1][r]);
        // lazy rescale: only when the row maximum grows by more than 2^kLazy (the same
        // decision in both halves: same m, same maximum)
        const bool grow = m != -INFINITY && mx > m + kLazy;
        if (__any_sync(0xffffffffu, grow)) {
          if (i >= 1 && !warp_wait(&sm.pv_done[u][(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), &sm.abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = grow ? ex2(m - mx) : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < 2; ++cc) {
            float v[32];
            tmem_ld32(lane_addr + o_col + cc * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= alpha;
            tmem_st32(lane_addr + o_col + cc * 32, v);
          }
          tmem_wait_st();
          if (grow) { l *= alpha; m = mx; }
        }
        if (m == -INFINITY) m = mx;                // first visible key of the row (O is zero)
        // subtrahend of the exponents: the running maximum, or +inf where the row sees none
        // of these keys (every weight 0)
        const float mu = lim < 0 ? INFINITY : (m == -INFINITY ? 0.f : m);
        uint32_t pw[16];                           // P (bf16 pairs) of this thread's 32 keys
        const unsigned long long sl2x2 = f2_pack(sl2, sl2), nmu2 = f2_pack(-mu, -mu);
        unsigned long long ps2[2] = {0ull, 0ull};  // two independent chains of packed sums
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          // 2^(x * log2(e)/sqrt(d) - mu) for a pair of keys; a masked key (-inf) gives 0
          float e0, e1;
          f2_unpack(f2_fma(f2_pack(x[2 * q], x[2 * q + 1]), sl2x2, nmu2), e0, e1);
          const float p0 = ex2(e0), p1 = ex2(e1);
          pw[q] = pack_bf16(p0, p1);
          ps2[q & 1] = f2_add(ps2[q & 1], f2_pack(p0, p1));   // the sums of the unrounded weights
        }
        {
          float a0, a1, b0, b1;
          f2_unpack(ps2[0], a0, a1);
          f2_unpack(ps2[1], b0, b1);
          l += (a0 + b0) + (a1 + b1);
        }
        // P over the first 16 of the 32 S columns this thread has read
        tmem_st16(lane_addr + (uint32_t)(j & 1) * 64 + s_col, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[u][j & 1]);
      }
      if (!ok) break;
      // epilogue: O / l of each valid row, the row sum from both halves (in the maxima slot
      // of the next entry's parity: both halves have read the last entry's maxima)
      sm.xmax[j & 1][u][hf][r] = l;
      if (!pair_sync()) { ok = false; break; }
      const float lr = sm.xmax[j & 1][u][0][r] + sm.xmax[j & 1][u][1][r];
      if (n >= 1 && !warp_wait(&sm.pv_done[u][(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), &sm.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      __nv_bfloat16* orow = a.O + (((int64_t)t.b * a.nq + qi) * a.Hq + h) * kD + hf * 64;
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
        if (n >= 1) {
          tmem_ld32(lane_addr + o_col + cc * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = 0.f;
        }
        if (valid) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o4;
            o4.x = pack_bf16(v[q * 8 + 0] * inv, v[q * 8 + 1] * inv);
            o4.y = pack_bf16(v[q * 8 + 2] * inv, v[q * 8 + 3] * inv);
            o4.z = pack_bf16(v[q * 8 + 4] * inv, v[q * 8 + 5] * inv);
            o4.w = pack_bf16(v[q * 8 + 6] * inv, v[q * 8 + 7] * inv);
            *reinterpret_cast<uint4*>(orow + cc * 32 + q * 8) = o4;
          }
        }
      }
      if (valid && hf == 0 && a.lse) a.lse[((int64_t)t.b * a.nq + qi) * a.Hq + h] =
          lr > 0.f ? (m + log2f(lr)) * 0.6931471805599453f : -INFINITY;
      // the sums of this tile are read before the next tile's epilogue writes them
      if (!pair_sync()) { ok = false; break; }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[u]);
    }
    if (!ok) give_up(sm, a.dev_status);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_free(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// union of a tile's leaf lists, one CTA per (tile, range of kRange chunk ids):
// every chunk some row selected (with the masks of those rows, 128 bits per sub-tile),
// chunk 0 (the first key) and each row's own chunk, in ascending id order
// ---------------------------------------------------------------------------

struct UnionArgs {
  int B, nq, Hq, Hkv, G, Qt, nqt;
  int64_t t_cap, nr;
  const int64_t* q_pos;
  const int* leaf_ids;
  const int* leaf_cnt;
  int leaf_cap;
  int* ent_ids;
  uint4* ent_mask;
  int* ent_cnt;
  int32_t* dev_status;
};

constexpr int kMaskWords = 4 * kSub;             // 32-bit words of a tile's row mask

__global__ void __launch_bounds__(256) prefill_union_kernel(UnionArgs a) {
  __shared__ uint32_t mask[kMaskWords][kRange];
  __shared__ uint32_t present[kRange / 32];
  __shared__ unsigned int wtot[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tile = blockIdx.x / a.nr, rg = blockIdx.x % a.nr;
  const int64_t unit = tile / a.nqt;
  const int q0 = (int)(tile % a.nqt) * kSub * a.Qt;
  const int b = (int)(unit / a.Hkv), hk = (int)(unit % a.Hkv);
  const int64_t lo = rg * kRange, hi = lo + kRange;
  const int sub_rows = a.Qt * a.G;
  for (int i = tid; i < kRange; i += 256) {
#pragma unroll
    for (int w = 0; w < kMaskWords; ++w) mask[w][i] = 0u;
  }
  if (tid < kRange / 32) present[tid] = 0u;
  __syncthreads();
  // row R of the tile: sub-tile R / 128, row R % 128 of it (query (R % 128) / G, head (R % 128) % G)
  auto row_query = [&](int R, int& qi, int& hh) -> bool {
    const int u = R >> 7, rr = R & 127;
    if (rr >= sub_rows) return false;
    qi = q0 + u * a.Qt + rr / a.G;
    hh = hk * a.G + rr % a.G;
    return qi < a.nq;
  };
  // chunk 0 and each valid row's own chunk
  for (int R = tid; R < kSub * 128; R += 256) {
    int qi, hh;
    if (!row_query(R, qi, hh)) continue;
    const int64_t t = a.q_pos[(int64_t)b * a.nq + qi];
    if (t < 0 || t >= a.t_cap) {
      if (rg == 0) set_status(a.dev_status, ZHA_ERR_INVALID_ARG);
      continue;
    }
    const int64_t cur = t / kLeaf;
    if (cur >= lo && cur < hi) atomicOr(&present[(cur - lo) >> 5], 1u << ((cur - lo) & 31));
    if (lo == 0) atomicOr(&present[0], 1u);
  }
  // selected chunks: warp w takes rows w, w + 8, ...
  for (int R = warp; R < kSub * 128; R += 8) {
    int qi, hh;
    if (!row_query(R, qi, hh)) continue;
    const int64_t t = a.q_pos[(int64_t)b * a.nq + qi];
    if (t < 0 || t >= a.t_cap) continue;
    const int64_t nvis = t / kLeaf;
    const int64_t qh = ((int64_t)b * a.nq + qi) * a.Hq + hh;
    const int* lst = a.leaf_ids + qh * a.leaf_cap;
    int cnt = a.leaf_cnt[qh];
    cnt = cnt < 0 ? 0 : (cnt > a.leaf_cap ? a.leaf_cap : cnt);
    const int x0 = warp_lower_bound(lst, cnt, lo);
    const int x1 = warp_lower_bound(lst, cnt, hi);
    for (int x = x0 + lane; x < x1; x += 32) {
      const int id = lst[x];
      // ids outside [lo, hi) mean an unsorted list; beyond n_vis an invisible chunk
      if (id < lo || id >= hi || id >= nvis) { set_status(a.dev_status, ZHA_ERR_INVALID_ARG); continue; }
      atomicOr(&mask[R >> 5][id - lo], 1u << (R & 31));
    }
  }
  __syncthreads();
  // ordered compaction: thread tid owns ids [4 tid, 4 tid + 4)
  constexpr int kPer = kRange / 256;
  unsigned int cntl = 0;
  bool on[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int i = tid * kPer + q;
    uint32_t any = (present[i >> 5] >> (i & 31)) & 1u;
#pragma unroll
    for (int w = 0; w < kMaskWords; ++w) any |= mask[w][i];
    on[q] = any != 0u;
    cntl += on[q];
  }
  unsigned int x = cntl;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  unsigned int before = 0, total = 0;
  for (int w = 0; w < 8; ++w) { if (w < warp) before += wtot[w]; total += wtot[w]; }
  before += x - cntl;
  const int64_t base = blockIdx.x * (int64_t)kRange;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    if (!on[q]) continue;
    const int i = tid * kPer + q;
    a.ent_ids[base + before] = (int)(lo + i);
#pragma unroll
    for (int u = 0; u < kSub; ++u)
      a.ent_mask[(base + before) * kSub + u] = make_uint4(mask[4 * u][i], mask[4 * u + 1][i], mask[4 * u + 2][i],
                                                          mask[4 * u + 3][i]);
    ++before;
  }
  if (tid == 0) a.ent_cnt[blockIdx.x] = (int)total;
}

}  // namespace qt

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

// Q [B, nq, Hq, 128] bf16 as a 4-D map with boxes of 64 dims x G heads x Qt queries x 1.
static bool make_q_map(CUtensorMap* map, const void* Q, int B, int nq, int Hq, int G, int Qt) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)Hq, (cuuint64_t)nq, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)Hq * kD * 2, (cuuint64_t)nq * Hq * kD * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)Qt, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(Q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

PrefillWs prefill_ws(const zha_geom& g, int nq, size_t base) {
  PrefillWs w{};
  const int G = g.Hq / g.Hkv;
  w.Qt = kPrefillRows / G;
  w.nqt = (nq + qt::kSub * w.Qt - 1) / (qt::kSub * w.Qt);
  w.tiles = (int64_t)g.B * g.Hkv * w.nqt;
  w.nr = (ncap_of(g, 1) + 1 + kRange - 1) / kRange;
  const size_t slots = (size_t)w.tiles * w.nr * kRange;
  size_t off = base;
  w.ent_ids = off;  off = align_up(off + slots * 4);
  w.ent_mask = off; off = align_up(off + slots * 16 * qt::kSub);
  w.ent_cnt = off;  off = align_up(off + (size_t)w.tiles * w.nr * 4);
  w.bytes = off;
  return w;
}

cudaError_t prefill_attention(const PrefillCall& c) {
  const zha_geom& g = *c.g;
  const PrefillWs w = prefill_ws(g, c.nq, 0);
  const int G = g.Hq / g.Hkv;
  qt::UnionArgs ua{};
  ua.B = g.B; ua.nq = c.nq; ua.Hq = g.Hq; ua.Hkv = g.Hkv; ua.G = G; ua.Qt = w.Qt; ua.nqt = (int)w.nqt;
  ua.t_cap = g.t_cap; ua.nr = w.nr; ua.q_pos = c.q_pos;
  ua.leaf_ids = c.leaf_ids; ua.leaf_cnt = c.leaf_cnt; ua.leaf_cap = c.leaf_cap;
  ua.ent_ids = (int*)(c.ws + w.ent_ids);
  ua.ent_mask = (uint4*)(c.ws + w.ent_mask);
  ua.ent_cnt = (int*)(c.ws + w.ent_cnt);
  ua.dev_status = c.dev_status;
  qt::prefill_union_kernel<<<(unsigned)(w.tiles * w.nr), 256, 0, c.stream>>>(ua);
  count_launch();
  cudaError_t e = launch_status("prefill_union_kernel");
  if (e != cudaSuccess) return e;

  CUtensorMap qm, km, vm;
  const int64_t units_kv = (int64_t)g.B * g.Hkv;
  if (!make_q_map(&qm, c.Q, g.B, c.nq, g.Hq, G, w.Qt) || !make_kv_map(&km, c.K, units_kv, g.t_cap) ||
      !make_kv_map(&vm, c.V, units_kv, g.t_cap)) {
    note_cuda_error(cudaErrorInvalidValue, "cuTensorMapEncodeTiled");
    return cudaErrorInvalidValue;
  }
  qt::Args a{};
  a.B = g.B; a.nq = c.nq; a.Hq = g.Hq; a.Hkv = g.Hkv; a.G = G; a.Qt = w.Qt; a.nqt = (int)w.nqt;
  a.t_cap = g.t_cap; a.nr = w.nr; a.tiles = w.tiles; a.q_pos = c.q_pos;
  a.ent_ids = ua.ent_ids; a.ent_mask = ua.ent_mask; a.ent_cnt = ua.ent_cnt;
  a.O = (__nv_bfloat16*)c.O; a.lse = c.lse; a.dev_status = c.dev_status;
  const size_t smem = sizeof(qt::Smem) + 1024;
  cudaFuncSetAttribute(qt::prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int64_t grid = w.tiles < sm_count() ? w.tiles : sm_count();
  trace_begin(ZHA_TRACE_ATTN, c.stream);
  qt::prefill_tc_kernel<<<(unsigned)grid, qt::kThreads, smem, c.stream>>>(qm, km, vm, a);
  trace_end(ZHA_TRACE_ATTN, c.stream);
  count_launch();
  return launch_status("prefill_tc_kernel");
}

}  // namespace zha
