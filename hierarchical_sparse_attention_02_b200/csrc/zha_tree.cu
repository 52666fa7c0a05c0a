// Tree construction and maintenance: leaf summaries, parent merges, token append.
//
// Leaf summary ("ZHA summary" page, Tree Construction; arXiv 2610.42112 §III-A):
//   s_rj = q_hat_r . k_j / sqrt(d),  F_r = LSE_j s_rj,  a_rj = exp(s_rj - F_r),
//   k_hat_r = sum_j a_rj k_j,  b_hat_r = F_r - q_hat_r . k_hat_r / sqrt(d).
// Parent merge (§III-B; App. D-B2, per-reference stable-state merge, no re-anchoring):
//   F_P = LSE_c F_c,  k_hat_P = sum_c exp(F_c - F_P) k_hat_c,  b_hat_P as above.
// All arithmetic is fp64 with fixed-order reductions, so a summary is bit-identical
// from run to run and agrees with an exact evaluation to ~1e-15 before it is stored
// (merge state fp32, routing k_hat in the KV dtype, b_hat fp32).  The kernels are
// templated on R so that the per-reference accumulators stay in registers.
#include "zha_internal.cuh"

namespace zha {

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
// leaf summaries: one CTA of 64 threads per leaf chunk (thread j <-> key j, then
// thread i <-> dims 2i, 2i+1)
// ---------------------------------------------------------------------------

template <typename KT, int R>
struct alignas(16) LeafSmem {
  KT keys[kLeaf][kD];           // the chunk, raw
  double qref[R][kD];           // reference queries in fp64
  double w[R][kLeaf];           // attention weights a_rj
  double red[2][R];             // cross-warp partials
  double Fr[R];
};

template <typename KT, int R>
__global__ void __launch_bounds__(64) leaf_summarize_kernel(
    const KT* __restrict__ K, const float* __restrict__ qref, int Hkv, int64_t t_cap,
    int64_t leaf_lo, int64_t nleaf, LevelPtrs out, double scale) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  LeafSmem<KT, R>& sm = *reinterpret_cast<LeafSmem<KT, R>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x / nleaf;          // b * Hkv + h
  const int64_t leaf = leaf_lo + blockIdx.x % nleaf;
  const int h = (int)(unit % Hkv);

  for (int i = tid; i < R * kD; i += 64) sm.qref[i / kD][i % kD] = (double)qref[(int64_t)h * R * kD + i];
  __syncthreads();

  // phase 1: scores of key j against every reference, streaming the key row once
  const KT* krow = K + (unit * t_cap + leaf * kLeaf + tid) * kD;
  double acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0;
  constexpr int kVec = 16 / sizeof(KT);
#pragma unroll 2
  for (int c = 0; c < kD; c += kVec) {
    const uint4 v = *reinterpret_cast<const uint4*>(krow + c);
    *reinterpret_cast<uint4*>(&sm.keys[tid][c]) = v;
    const KT* e = reinterpret_cast<const KT*>(&v);
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const double x = to_f64(e[u]);
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fma(sm.qref[r][c + u], x, acc[r]);
    }
  }
  // per-reference max over the 64 keys (fixed-order tree over lanes, then warps)
  double m[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    acc[r] *= scale;
    double v = acc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, shfl_xor_f64(v, o));
    m[r] = v;
  }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) sm.red[warp][r] = m[r];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) m[r] = fmax(sm.red[0][r], sm.red[1][r]);
  __syncthreads();
  // exponentials and their sum
  double e[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    e[r] = exp(acc[r] - m[r]);
    double v = e[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += shfl_xor_f64(v, o);
    if (lane == 0) sm.red[warp][r] = v;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const double Z = sm.red[0][r] + sm.red[1][r];
    sm.w[r][tid] = e[r] / Z;
    if (tid == 0) sm.Fr[r] = m[r] + log(Z);
  }
  __syncthreads();

  // phase 2: k_hat_r[2i, 2i+1] = sum_j a_rj k_j
  double k0[R], k1[R];
#pragma unroll
  for (int r = 0; r < R; ++r) k0[r] = k1[r] = 0.0;
#pragma unroll 4
  for (int j = 0; j < kLeaf; ++j) {
    const double x0 = to_f64(sm.keys[j][2 * tid]);
    const double x1 = to_f64(sm.keys[j][2 * tid + 1]);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const double a = sm.w[r][j];
      k0[r] = fma(a, x0, k0[r]);
      k1[r] = fma(a, x1, k1[r]);
    }
  }
  // b_hat_r = F_r - scale * q_hat_r . k_hat_r
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    double v = fma(sm.qref[r][2 * tid], k0[r], sm.qref[r][2 * tid + 1] * k1[r]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += shfl_xor_f64(v, o);
    if (lane == 0) sm.red[warp][r] = v;
  }
  __syncthreads();
  const int64_t node = unit * out.n_cap + leaf;
  KT* kr = reinterpret_cast<KT*>(out.k_route) + node * R * kD;
  float* ks = out.k_state + node * R * kD;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    kr[r * kD + 2 * tid] = from_f64<KT>(k0[r]);
    kr[r * kD + 2 * tid + 1] = from_f64<KT>(k1[r]);
    *reinterpret_cast<float2*>(ks + r * kD + 2 * tid) =
        make_float2(__double2float_rn(k0[r]), __double2float_rn(k1[r]));
  }
  if (tid < R) {
    const double F = sm.Fr[tid];
    const double qk = sm.red[0][tid] + sm.red[1][tid];
    out.F[node * R + tid] = __double2float_rn(F);
    out.b_hat[node * R + tid] = __double2float_rn(F - scale * qk);
  }
}

// ---------------------------------------------------------------------------
// parent merge: one CTA of 128 threads per parent node (thread <-> dim)
// ---------------------------------------------------------------------------

constexpr int kMaxBranch = 64;

template <typename KT, int R>
__global__ void __launch_bounds__(128) parent_merge_kernel(
    const float* __restrict__ qref, int Hkv, int branch, int64_t lo, int64_t n,
    LevelPtrs child, LevelPtrs out, double scale) {
  __shared__ double Fc[kMaxBranch][R];
  __shared__ double w[kMaxBranch][R];
  __shared__ double Fp[R];
  __shared__ double red[4][R];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t unit = blockIdx.x / n;
  const int64_t node = lo + blockIdx.x % n;
  const int h = (int)(unit % Hkv);
  const int64_t c0 = unit * child.n_cap + node * branch;   // first child entry
  for (int i = tid; i < branch * R; i += 128) {
    const int c = i / R, r = i % R;
    Fc[c][r] = (double)child.F[(c0 + c) * R + r];
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
    double v = (double)qref[((int64_t)h * R + r) * kD + tid] * acc[r];
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
// host drivers
// ---------------------------------------------------------------------------

template <typename KT, int R>
static cudaError_t launch_leaves(const zha_geom& g, const TreeLayout& L, const void* K,
                                 const float* qref, void* tree, int64_t lo, int64_t hi,
                                 cudaStream_t s) {
  const int64_t n = hi - lo;
  const int64_t blocks = (int64_t)g.B * g.Hkv * n;
  const size_t smem = sizeof(LeafSmem<KT, R>);
  cudaFuncSetAttribute(leaf_summarize_kernel<KT, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  leaf_summarize_kernel<KT, R><<<(unsigned)blocks, 64, smem, s>>>(
      (const KT*)K, qref, g.Hkv, g.t_cap, lo, n, level_ptrs(g, L, tree, 1), 1.0 / sqrt((double)g.d));
  count_launch();
  return launch_status("leaf_summarize_kernel");
}

template <typename KT, int R>
static cudaError_t launch_merge(const zha_geom& g, const TreeLayout& L, const float* qref,
                                void* tree, int level, int64_t lo, int64_t hi, cudaStream_t s) {
  const int64_t n = hi - lo;
  const int64_t blocks = (int64_t)g.B * g.Hkv * n;
  parent_merge_kernel<KT, R><<<(unsigned)blocks, 128, 0, s>>>(
      qref, g.Hkv, g.branch, lo, n, level_ptrs(g, L, tree, level - 1), level_ptrs(g, L, tree, level),
      1.0 / sqrt((double)g.d));
  count_launch();
  return launch_status("parent_merge_kernel");
}

template <typename KT, int R>
static cudaError_t extend_t(const zha_geom& g, const TreeLayout& L, const void* K, const float* qref,
                            void* tree, int64_t t_old, int64_t t_new, cudaStream_t s) {
  for (int l = 1; l <= g.depth; ++l) {
    const int64_t span = span_of(g, l);
    const int64_t lo = t_old / span, hi = t_new / span;
    if (hi <= lo) break;   // nothing completes at this level, nor above
    const cudaError_t e = l == 1 ? launch_leaves<KT, R>(g, L, K, qref, tree, lo, hi, s)
                                 : launch_merge<KT, R>(g, L, qref, tree, l, lo, hi, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename KT>
static cudaError_t extend_r(const zha_geom& g, const TreeLayout& L, const void* K, const float* qref,
                            void* tree, int64_t t_old, int64_t t_new, cudaStream_t s) {
  switch (g.R) {
    case 1: return extend_t<KT, 1>(g, L, K, qref, tree, t_old, t_new, s);
    case 2: return extend_t<KT, 2>(g, L, K, qref, tree, t_old, t_new, s);
    case 4: return extend_t<KT, 4>(g, L, K, qref, tree, t_old, t_new, s);
    case 8: return extend_t<KT, 8>(g, L, K, qref, tree, t_old, t_new, s);
    case 16: return extend_t<KT, 16>(g, L, K, qref, tree, t_old, t_new, s);
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
