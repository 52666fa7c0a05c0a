// Tree construction and maintenance: leaf summaries, parent merges, token append.
//
// Leaf summary ("ZHA summary" page, Tree Construction; arXiv 2610.42112 §III-A):
//   s_rj = q_hat_r . k_j / sqrt(d),  F_r = LSE_j s_rj,  a_rj = exp(s_rj - F_r),
//   k_hat_r = sum_j a_rj k_j,  b_hat_r = F_r - q_hat_r . k_hat_r / sqrt(d).
// Parent merge (§III-B; App. D-B2, per-reference stable-state merge, no re-anchoring):
//   F_P = LSE_c F_c,  k_hat_P = sum_c exp(F_c - F_P) k_hat_c,  b_hat_P as above.
// Rotary positions (§III-B, models with RoPE; geometry rope_pairs = h > 0, the h rotary
// frequencies f_i stored after the reference queries): a node's references are rotated to
// its last key position P, dims (i, i + h) by the angle P * f_i, and before a merge each
// child's log mass moves to the parent's rotated reference along its tangent plane,
//   F_c += <k_hat_c, q_hat_P - q_hat_c> / sqrt(d).
// All arithmetic is fp64 with fixed-order reductions, so a summary is bit-identical
// from run to run and agrees with an exact evaluation to ~1e-15 before it is stored
// (merge state fp32, routing k_hat in the KV dtype, b_hat fp32).  The kernels are
// templated on R so that the per-reference accumulators stay in registers.
#include "zha_internal.cuh"

namespace zha {

// Element `dim` of reference row q (fp32, d values) rotated by the angles whose cosines and
// sines are cs[i], sn[i] (i < h): dims i < h take x_i cos - x_{i+h} sin, dims h <= i < 2h
// take x_i cos + x_{i-h} sin, the rest pass through.  Each product and the sum are rounded
// separately (no fused multiply-add), the order of the plain formula.
// rope_one: the same for one element, given the cosine and sine of its pair's angle.
__device__ __forceinline__ double rope_one(const float* q, int dim, int h, double c, double s) {
  const double x = (double)q[dim];
  if (dim < h) return __dsub_rn(__dmul_rn(x, c), __dmul_rn((double)q[dim + h], s));
  if (dim < 2 * h) return __dadd_rn(__dmul_rn(x, c), __dmul_rn((double)q[dim - h], s));
  return x;
}

__device__ __forceinline__ double rope_elem(const float* q, int dim, int h, const double* cs,
                                            const double* sn) {
  const int j = dim < h ? dim : dim - h;             // the pair of dim (unused past 2h)
  return dim < 2 * h ? rope_one(q, dim, h, cs[j], sn[j]) : (double)q[dim];
}

struct LevelPtrs {
  void* k_route;
  float* b_hat;
  float* F;
  float* k_state;
  int64_t n_cap;
};

inline LevelPtrs level_ptrs(const zha_geom& g, const TreeLayout& L, void* base, int level) {
  char* b = (char*)base;
  const zha_level_layout& lv = L.lv[level];
  return LevelPtrs{b + lv.k_route_off, (float*)(b + lv.b_hat_off), (float*)(b + lv.F_off),
                   (float*)(b + lv.k_state_off), lv.n_cap};
}

// ---------------------------------------------------------------------------
// leaf summaries on the fp64 tensor cores: one CTA of 4 warps per leaf chunk.
//   phase 1  S^T[64 keys x R] = K[64 x 128] . q_hat^T      (mma.m8n8k4.f64, 8 keys per tile)
//   softmax  per reference over the 64 keys (fixed-order warp reductions)
//   phase 2  k_hat^T[128 x R] = K^T[128 x 64] . a^T        (8 dims per tile, 4 keys per step)
// References are padded to a multiple of 8 (the mma's N); the padding columns are zero.
// In phase 1 lane L holds A[key L/4][dim 32*(L%4) + s] at k-step s: 32 contiguous dims of its
// key; the B fragments (q_hat, then a) sit in shared memory as [step][lane].
// ---------------------------------------------------------------------------

template <typename KT, int R>
struct alignas(16) LeafTcSmem {
  static constexpr int NT = (R + 7) / 8;             // N-tiles of references
  static constexpr int kRow = kD + 16 / sizeof(KT) * (sizeof(KT) == 2 ? 1 : 2);  // padded row
  KT keys[kLeaf][kRow];                              // first: 16-byte aligned rows (272 / 544 B)
  double qf[NT][32][32];                             // q_hat B fragments: [tile][step][lane]
  double af[NT][16][32];                             // a B fragments:     [tile][step][lane]
  double sS[R][kLeaf];                               // scaled scores
  double Fr[R];
  double red[4][R];                                  // per-warp q_hat . k_hat partials
};

template <typename KT, int R, bool ROPE>
__global__ void __launch_bounds__(128) leaf_summarize_tc_kernel(
    const KT* __restrict__ K, const float* __restrict__ qref, int Hkv, int64_t t_cap,
    int64_t leaf_lo, int64_t nleaf, LevelPtrs out, double scale, int rope_pairs) {
  using Sm = LeafTcSmem<KT, R>;
  constexpr int NT = Sm::NT;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Sm& sm = *reinterpret_cast<Sm*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x / nleaf;           // b * Hkv + h
  const int64_t leaf = leaf_lo + blockIdx.x % nleaf;
  const int h = (int)(unit % Hkv);
  const float* q = qref + (int64_t)h * R * kD;
  if constexpr (ROPE) {
    // the references rotated to the leaf's last key
    __shared__ double cs[kD / 2], sn[kD / 2];
    const float* freq = qref + (int64_t)Hkv * R * kD;
    const double pos = (double)((leaf + 1) * kLeaf - 1);
    if (tid < rope_pairs) sincos(pos * (double)freq[tid], &sn[tid], &cs[tid]);
    __syncthreads();
    for (int i = tid; i < NT * 32 * 32; i += 128) {
      const int nt = i / 1024, s = (i / 32) % 32, L = i % 32;
      const int r = nt * 8 + (L >> 2);
      sm.qf[nt][s][L] = r < R ? rope_elem(q + r * kD, 32 * (L & 3) + s, rope_pairs, cs, sn) : 0.0;
    }
  } else {
    for (int i = tid; i < NT * 32 * 32; i += 128) {
      const int nt = i / 1024, s = (i / 32) % 32, L = i % 32;
      const int r = nt * 8 + (L >> 2);
      sm.qf[nt][s][L] = r < R ? (double)q[r * kD + 32 * (L & 3) + s] : 0.0;
    }
  }
  __syncthreads();

  // phase 1: warp w takes keys [16w, 16w + 16) as two tiles of 8, interleaved (two
  // independent accumulator chains per tile and reference tile)
  constexpr int kVec = 16 / sizeof(KT);
  constexpr int kNv = 32 / kVec;
  const KT* kbase = K + (unit * t_cap + leaf * kLeaf) * kD;
  uint4 v[2][kNv];
#pragma unroll
  for (int tile = 0; tile < 2; ++tile) {
    const int key = warp * 16 + tile * 8 + (lane >> 2);
    const uint4* src = reinterpret_cast<const uint4*>(kbase + key * kD + 32 * (lane & 3));
#pragma unroll
    for (int i = 0; i < kNv; ++i) v[tile][i] = __ldg(src + i);
  }
#pragma unroll
  for (int tile = 0; tile < 2; ++tile) {
    const int key = warp * 16 + tile * 8 + (lane >> 2);
#pragma unroll
    for (int i = 0; i < kNv; ++i)
      *reinterpret_cast<uint4*>(&sm.keys[key][32 * (lane & 3) + i * kVec]) = v[tile][i];
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    double c[2][2][2] = {};                          // [tile][chain][d0/d1]
#pragma unroll
    for (int s = 0; s < 32; ++s) {
      const double b = sm.qf[nt][s][lane];
#pragma unroll
      for (int tile = 0; tile < 2; ++tile) {
        mma_f64(c[tile][s & 1][0], c[tile][s & 1][1], (double)u4_elem<KT>(v[tile][s / kVec], s % kVec), b);
      }
    }
    const int r0 = nt * 8 + 2 * (lane & 3);
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
      const int krow = warp * 16 + tile * 8 + (lane >> 2);
      if (r0 < R) sm.sS[r0][krow] = (c[tile][0][0] + c[tile][1][0]) * scale;
      if (r0 + 1 < R) sm.sS[r0 + 1][krow] = (c[tile][0][1] + c[tile][1][1]) * scale;
    }
  }
  __syncthreads();

  // softmax of each reference over the 64 keys: warp w takes references w, w + 4, ...
  for (int r = warp; r < R; r += 4) {
    const double v0 = sm.sS[r][lane], v1 = sm.sS[r][lane + 32];
    double m = fmax(v0, v1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, shfl_xor_f64(m, o));
    const double e0 = exp(v0 - m), e1 = exp(v1 - m);
    double z = e0 + e1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += shfl_xor_f64(z, o);
    if (lane == 0) sm.Fr[r] = m + log(z);
    // a[r][key] -> B fragment of phase 2: step key / 4, lane (r % 8) * 4 + key % 4
    sm.af[r / 8][lane >> 2][(r & 7) * 4 + (lane & 3)] = e0 / z;
    sm.af[r / 8][(lane + 32) >> 2][(r & 7) * 4 + (lane & 3)] = e1 / z;
  }
  for (int i = tid; i < NT * 16 * 32; i += 128) {      // zero the padding references
    const int nt = i / 512, s = (i / 32) % 16, L = i % 32;
    if (nt * 8 + (L >> 2) >= R) sm.af[nt][s][L] = 0.0;
  }
  __syncthreads();

  // phase 2: warp w takes the dim tiles w, w + 4, w + 8, w + 12
  const int64_t node = unit * out.n_cap + leaf;
  KT* kr = reinterpret_cast<KT*>(out.k_route) + node * R * kD;
  float* ks = out.k_state + node * R * kD;
  double qk[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) qk[nt][0] = qk[nt][1] = 0.0;
  double c4[4][NT][2] = {};                          // the warp's 4 dim tiles, interleaved
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    double b[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) b[nt] = sm.af[nt][s][lane];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
      const double av = (double)to_f32(sm.keys[4 * s + (lane & 3)][(warp + 4 * mi) * 8 + (lane >> 2)]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f64(c4[mi][nt][0], c4[mi][nt][1], av, b[nt]);
    }
  }
#pragma unroll
  for (int mi = 0; mi < 4; ++mi) {
    const int mt = warp + 4 * mi;
    const int dim = mt * 8 + (lane >> 2);
    double (&c)[NT][2] = c4[mi];
    // lane holds k_hat[dim][refs nt*8 + 2*(lane%4) + {0, 1}]
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int r = nt * 8 + 2 * (lane & 3) + x;
        if (r < R) {
          kr[r * kD + dim] = from_f64<KT>(c[nt][x]);
          ks[r * kD + dim] = __double2float_rn(c[nt][x]);
          // q_hat[r][dim] from the phase-1 fragments: step dim % 32, lane (r % 8) * 4 + dim / 32
          qk[nt][x] = fma(sm.qf[nt][dim & 31][(r & 7) * 4 + (dim >> 5)], c[nt][x], qk[nt][x]);
        }
      }
    }
  }
  // b_hat_r = F_r - scale * q_hat_r . k_hat_r: lanes with the same lane % 4 hold one reference
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      double v = qk[nt][x];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) v += shfl_xor_f64(v, o);
      const int r = nt * 8 + 2 * (lane & 3) + x;
      if (lane < 4 && r < R) sm.red[warp][r] = v;
    }
  }
  __syncthreads();
  if (tid < R) {
    const double F = sm.Fr[tid];
    const double qkt = (sm.red[0][tid] + sm.red[1][tid]) + (sm.red[2][tid] + sm.red[3][tid]);
    out.F[node * R + tid] = __double2float_rn(F);
    out.b_hat[node * R + tid] = __double2float_rn(F - scale * qkt);
  }
}

// ---------------------------------------------------------------------------
// parent merge: one CTA of 128 threads per parent node (thread <-> dim)
// ---------------------------------------------------------------------------

constexpr int kMaxBranch = 64;

template <typename KT, int R, bool ROPE>
__global__ void __launch_bounds__(128) parent_merge_kernel(
    const float* __restrict__ qref, int Hkv, int branch, int64_t lo, int64_t n,
    LevelPtrs child, LevelPtrs out, double scale, int rope_pairs, int64_t span_c) {
  __shared__ double Fc[kMaxBranch][R];
  __shared__ double w[kMaxBranch][R];
  __shared__ double Fp[R];
  __shared__ double red[4][R];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x / n;
  const int64_t node = lo + blockIdx.x % n;
  const int h = (int)(unit % Hkv);
  const int64_t c0 = unit * child.n_cap + node * branch;   // first child entry
  const float* qh = qref + (int64_t)h * R * kD;
  for (int i = tid; i < branch * R; i += 128) {
    const int c = i / R, r = i % R;
    Fc[c][r] = (double)child.F[(c0 + c) * R + r];
  }
  // with rotation: this thread's element (dim = tid) of every rotated parent reference
  double qp[ROPE ? R : 1];
  if constexpr (ROPE) {
    __shared__ double cr[2][4][R];                         // per-warp partials, double-buffered
    const float* freq = qref + (int64_t)Hkv * R * kD;
    const int j = tid < rope_pairs ? tid : (tid < 2 * rope_pairs ? tid - rope_pairs : -1);
    const double f = j >= 0 ? (double)freq[j] : 0.0;
    double c = 1.0, sv = 0.0;
    if (j >= 0) sincos((double)((node + 1) * span_c * branch - 1) * f, &sv, &c);
#pragma unroll
    for (int r = 0; r < R; ++r) qp[r] = rope_one(qh + r * kD, tid, rope_pairs, c, sv);
    __syncthreads();                                       // Fc is loaded
    // re-anchor each child: F_c += scale * <k_hat_c, q_hat_P - q_hat_c>
    for (int ci = 0; ci < branch; ++ci) {
      double cc = 1.0, sc = 0.0;
      if (j >= 0) sincos((double)((node * branch + ci + 1) * span_c - 1) * f, &sc, &cc);
      const float* ks = child.k_state + (c0 + ci) * R * kD;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const double diff = j >= 0 ? qp[r] - rope_one(qh + r * kD, tid, rope_pairs, cc, sc) : 0.0;
        double v = j >= 0 ? (double)ks[r * kD + tid] * diff : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += shfl_xor_f64(v, o);
        if (lane == 0) cr[ci & 1][warp][r] = v;
      }
      __syncthreads();
      if (tid < R)
        Fc[ci][tid] += scale * ((cr[ci & 1][0][tid] + cr[ci & 1][1][tid]) + (cr[ci & 1][2][tid] + cr[ci & 1][3][tid]));
    }
  }
  __syncthreads();
  // F_P = LSE_c F_c (one thread per reference, children in order)
  if (tid < R) {
    double M = -INFINITY;
    for (int c = 0; c < branch; ++c) M = fmax(M, Fc[c][tid]);
    double Z = 0.0;
    for (int c = 0; c < branch; ++c) Z += exp(Fc[c][tid] - M);
    Fp[tid] = M + log(Z);
  }
  __syncthreads();
  // merge weights w_cr = exp(F_cr - F_P)
  for (int i = tid; i < branch * R; i += 128) {
    const int c = i / R, r = i % R;
    w[c][r] = exp(Fc[c][r] - Fp[r]);
  }
  __syncthreads();
  double acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0;
  for (int c = 0; c < branch; ++c) {
    const float* ks = child.k_state + (c0 + c) * R * kD;
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = fma(w[c][r], (double)ks[r * kD + tid], acc[r]);
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    double v = (ROPE ? qp[ROPE ? r : 0] : (double)qh[r * kD + tid]) * acc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += shfl_xor_f64(v, o);
    if (lane == 0) red[warp][r] = v;
  }
  __syncthreads();
  const int64_t pn = unit * out.n_cap + node;
  KT* kr = reinterpret_cast<KT*>(out.k_route) + pn * R * kD;
  float* ks = out.k_state + pn * R * kD;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    kr[r * kD + tid] = from_f64<KT>(acc[r]);
    ks[r * kD + tid] = __double2float_rn(acc[r]);
  }
  if (tid < R) {
    const double qk = (red[0][tid] + red[1][tid]) + (red[2][tid] + red[3][tid]);
    out.F[pn * R + tid] = __double2float_rn(Fp[tid]);
    out.b_hat[pn * R + tid] = __double2float_rn(Fp[tid] - scale * qk);
  }
}

// ---------------------------------------------------------------------------
// append: [B, n_new, Hkv, d] -> [B, Hkv, t_cap, d] at positions [t_old, t_old + n_new)
// ---------------------------------------------------------------------------

__global__ void append_kv_kernel(uint4* __restrict__ K, uint4* __restrict__ V,
                                 const uint4* __restrict__ kn, const uint4* __restrict__ vn,
                                 int Hkv, int n_new, int64_t t_cap, int64_t t_old, int vec_per_row,
                                 int64_t total_vec) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total_vec;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / vec_per_row;       // (b, tok, h)
    const int c = (int)(i % vec_per_row);
    const int h = (int)(row % Hkv);
    const int64_t tok = (row / Hkv) % n_new;
    const int64_t b = row / ((int64_t)Hkv * n_new);
    const int64_t dst = (((b * Hkv + h) * t_cap) + t_old + tok) * vec_per_row + c;
    K[dst] = kn[i];
    V[dst] = vn[i];
  }
}

// ---------------------------------------------------------------------------
// host side: the launches of a tree extension
// ---------------------------------------------------------------------------

template <typename KT, int R, bool ROPE>
static cudaError_t launch_leaves(const zha_geom& g, const TreeLayout& L, const void* K,
                                 const float* qref, void* tree, int64_t lo, int64_t hi,
                                 cudaStream_t s) {
  const int64_t n = hi - lo;
  const int64_t blocks = (int64_t)g.B * g.Hkv * n;
  const size_t smem = sizeof(LeafTcSmem<KT, R>);
  cudaFuncSetAttribute(leaf_summarize_tc_kernel<KT, R, ROPE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  leaf_summarize_tc_kernel<KT, R, ROPE><<<(unsigned)blocks, 128, smem, s>>>(
      (const KT*)K, qref, g.Hkv, g.t_cap, lo, n, level_ptrs(g, L, tree, 1), 1.0 / sqrt((double)g.d),
      g.rope_pairs);
  count_launch();
  return launch_status("leaf_summarize_tc_kernel");
}

template <typename KT, int R, bool ROPE>
static cudaError_t launch_merge(const zha_geom& g, const TreeLayout& L, const float* qref,
                                void* tree, int level, int64_t lo, int64_t hi, cudaStream_t s) {
  const int64_t n = hi - lo;
  const int64_t blocks = (int64_t)g.B * g.Hkv * n;
  parent_merge_kernel<KT, R, ROPE><<<(unsigned)blocks, 128, 0, s>>>(
      qref, g.Hkv, g.branch, lo, n, level_ptrs(g, L, tree, level - 1), level_ptrs(g, L, tree, level),
      1.0 / sqrt((double)g.d), g.rope_pairs, span_of(g, level - 1));
  count_launch();
  return launch_status("parent_merge_kernel");
}

template <typename KT, int R, bool ROPE>
static cudaError_t extend_t(const zha_geom& g, const TreeLayout& L, const void* K, const float* qref,
                            void* tree, int64_t t_old, int64_t t_new, cudaStream_t s) {
  for (int l = 1; l <= g.depth; ++l) {
    const int64_t span = span_of(g, l);
    const int64_t lo = t_old / span, hi = t_new / span;
    if (hi <= lo) break;   // nothing completes at this level, nor above
    const cudaError_t e = l == 1 ? launch_leaves<KT, R, ROPE>(g, L, K, qref, tree, lo, hi, s)
                                 : launch_merge<KT, R, ROPE>(g, L, qref, tree, l, lo, hi, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename KT, int R>
static cudaError_t extend_rope(const zha_geom& g, const TreeLayout& L, const void* K, const float* qref,
                               void* tree, int64_t t_old, int64_t t_new, cudaStream_t s) {
  return g.rope_pairs > 0 ? extend_t<KT, R, true>(g, L, K, qref, tree, t_old, t_new, s)
                          : extend_t<KT, R, false>(g, L, K, qref, tree, t_old, t_new, s);
}

template <typename KT>
static cudaError_t extend_r(const zha_geom& g, const TreeLayout& L, const void* K, const float* qref,
                            void* tree, int64_t t_old, int64_t t_new, cudaStream_t s) {
  switch (g.R) {
    case 1: return extend_rope<KT, 1>(g, L, K, qref, tree, t_old, t_new, s);
    case 2: return extend_rope<KT, 2>(g, L, K, qref, tree, t_old, t_new, s);
    case 4: return extend_rope<KT, 4>(g, L, K, qref, tree, t_old, t_new, s);
    case 8: return extend_rope<KT, 8>(g, L, K, qref, tree, t_old, t_new, s);
    case 16: return extend_rope<KT, 16>(g, L, K, qref, tree, t_old, t_new, s);
    default: return cudaErrorInvalidValue;   // zha_check_geom admits powers of two only
  }
}

// Summarise every node completed when the cache grows from t_old to t_new keys.
cudaError_t tree_extend(const zha_geom& g, const void* K, const float* qref, void* tree,
                        int64_t t_old, int64_t t_new, cudaStream_t s) {
  const TreeLayout L = tree_layout(g);
  return g.dtype == ZHA_BF16 ? extend_r<__nv_bfloat16>(g, L, K, qref, tree, t_old, t_new, s)
                             : extend_r<float>(g, L, K, qref, tree, t_old, t_new, s);
}

cudaError_t append_tokens(const zha_geom& g, void* K, void* V, const void* k_new,
                          const void* v_new, int64_t t_old, int n_new, cudaStream_t s) {
  if (n_new <= 0) return cudaSuccess;
  const int vec_per_row = g.d * elem_bytes(g) / 16;
  const int64_t total = (int64_t)g.B * n_new * g.Hkv * vec_per_row;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  append_kv_kernel<<<(unsigned)blocks, threads, 0, s>>>((uint4*)K, (uint4*)V, (const uint4*)k_new,
                                                        (const uint4*)v_new, g.Hkv, n_new, g.t_cap,
                                                        t_old, vec_per_row, total);
  count_launch();
  return launch_status("append_kv_kernel");
}

}  // namespace zha
