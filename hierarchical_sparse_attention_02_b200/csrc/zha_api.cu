// The C ABI declared in include/zha.h: argument validation, buffer sizing and the
// composition of the kernels into the calls of the hot path.
#include <math.h>
#include <stdio.h>

#include "zha_internal.cuh"

namespace zha {

std::atomic<int64_t> g_launches{0};
Tracer g_trace[5];

static char g_last_error[256] = "no error";

void note_cuda_error(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

static zha_status from_cuda(cudaError_t e) { return e == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA; }

static bool valid_p(double p) { return p > 0.0 && p <= 1.0 && !isnan(p); }

// The workspace check of every entry point: sizes whose arrays would not fit 64-bit byte
// counts are unsupported (zha_workspace_bytes returns 0 for them), smaller buffers too small.
static zha_status check_ws(const zha_geom* g, int32_t nq, int32_t op, const zha_buf& ws) {
  const size_t need = zha_workspace_bytes(g, nq, op);
  if (need == 0) return ZHA_ERR_UNSUPPORTED;
  return ws.bytes < need ? ZHA_ERR_CAPACITY : ZHA_OK;
}

}  // namespace zha

using namespace zha;

extern "C" {

const char* zha_status_str(int32_t s) {
  switch (s) {
    case ZHA_OK: return "ok";
    case ZHA_ERR_INVALID_ARG: return "invalid argument";
    case ZHA_ERR_UNSUPPORTED: return "unsupported geometry or dtype";
    case ZHA_ERR_CAPACITY: return "capacity exceeded";
    case ZHA_ERR_CUDA: return "CUDA launch error";
    case ZHA_ERR_DEVICE: return "device-side error";
    default: return "unknown status";
  }
}

zha_status zha_check_geom(const zha_geom* g) {
  if (!g) return ZHA_ERR_INVALID_ARG;
  if (g->B < 1 || g->Hq < 1 || g->Hkv < 1 || g->R < 1 || g->depth < 1 || g->t_cap < 1)
    return ZHA_ERR_INVALID_ARG;
  if (g->Hq % g->Hkv != 0) return ZHA_ERR_INVALID_ARG;
  if (g->rope_pairs < 0 || g->rope_pairs > g->d / 2) return ZHA_ERR_INVALID_ARG;
  if (g->d != kD || g->leaf != kLeaf) return ZHA_ERR_UNSUPPORTED;
  if (g->Hq / g->Hkv > kMaxG || g->R > kMaxR || g->depth > kMaxDepth) return ZHA_ERR_UNSUPPORTED;
  if (g->R & (g->R - 1)) return ZHA_ERR_UNSUPPORTED;     // R in {1, 2, 4, 8, 16}
  if (g->branch < 2 || g->branch > 64) return ZHA_ERR_UNSUPPORTED;
  if (g->dtype != ZHA_F32 && g->dtype != ZHA_BF16) return ZHA_ERR_UNSUPPORTED;
  if (g->t_cap % kLeaf != 0) return ZHA_ERR_INVALID_ARG;
  if (g->t_cap / kLeaf + 2 > (int64_t)INT32_MAX / 2) return ZHA_ERR_UNSUPPORTED;
  if (!cache_fits(*g)) return ZHA_ERR_UNSUPPORTED;
  return ZHA_OK;
}

size_t zha_tree_bytes(const zha_geom* g) {
  if (zha_check_geom(g) != ZHA_OK) return 0;
  return tree_layout(*g).bytes;
}

zha_status zha_tree_level(const zha_geom* g, int32_t level, zha_level_layout* out) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!out || level < 1 || level > g->depth) return ZHA_ERR_INVALID_ARG;
  *out = tree_layout(*g).lv[level];
  return ZHA_OK;
}

int64_t zha_leaf_cap(const zha_geom* g) {
  if (zha_check_geom(g) != ZHA_OK) return 0;
  return g->t_cap / g->leaf;
}

size_t zha_workspace_bytes(const zha_geom* g, int32_t nq, int32_t op) {
  if (zha_check_geom(g) != ZHA_OK || nq < 1 || !call_fits(*g, nq)) return 0;
  switch (op) {
    case ZHA_OP_ROUTE: return route_ws(*g, nq).bytes;
    case ZHA_OP_ATTN:
    case ZHA_OP_DENSE: return attn_ws(*g, nq).bytes;
    case ZHA_OP_PREFILL: return prefill_ws(*g, nq).bytes;
    case ZHA_OP_DECODE:
    case ZHA_OP_FLAT: {
      const size_t r = route_ws(*g, nq).bytes;
      const size_t a = attn_ws(*g, nq).bytes;
      return r > a ? r : a;   // routing finishes before the attention plan is built
    }
    default: return 0;
  }
}

int64_t zha_launch_count(void) { return g_launches.load(); }

const char* zha_last_error(void) { return g_last_error; }

void zha_trace(int32_t which, void* const* start, void* const* stop, int32_t n) {
  if (which < 1 || which > 4) return;
  Tracer& t = g_trace[which];
  t.start = start;
  t.stop = stop;
  t.n = (start && stop && n > 0) ? n : 0;
  t.done = 0;
}

int32_t zha_trace_count(int32_t which) { return (which >= 1 && which <= 4) ? g_trace[which].done : 0; }

zha_status zha_build_tree(const zha_geom* g, const void* K, int64_t T, const float* qref,
                          zha_buf tree, int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!K || !qref || !tree.base || !dev_status) return ZHA_ERR_INVALID_ARG;
  if (T < 0 || T > g->t_cap) return ZHA_ERR_INVALID_ARG;
  if (tree.bytes < zha_tree_bytes(g)) return ZHA_ERR_CAPACITY;
  return from_cuda(tree_extend(*g, K, qref, tree.base, 0, T, (cudaStream_t)stream));
}

zha_status zha_append(const zha_geom* g, void* K, void* V, const void* k_new, const void* v_new,
                      int64_t t_old, int32_t n_new, const float* qref, zha_buf tree,
                      int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!K || !V || !k_new || !v_new || !qref || !tree.base || !dev_status) return ZHA_ERR_INVALID_ARG;
  if (t_old < 0 || n_new < 0 || t_old + n_new > g->t_cap) return ZHA_ERR_INVALID_ARG;
  if (tree.bytes < zha_tree_bytes(g)) return ZHA_ERR_CAPACITY;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = append_tokens(*g, K, V, k_new, v_new, t_old, n_new, st);
  if (e != cudaSuccess) return ZHA_ERR_CUDA;
  return from_cuda(tree_extend(*g, K, qref, tree.base, t_old, t_old + n_new, st));
}

zha_status zha_route(const zha_geom* g, const void* Q, const int64_t* q_pos, int32_t nq, double p,
                     zha_buf tree, int32_t* leaf_ids, int32_t* leaf_cnt, int32_t leaf_cap,
                     int32_t* level_cnt, int32_t* level_ids, zha_buf ws, int32_t* dev_status,
                     void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!Q || !q_pos || nq < 1 || !valid_p(p) || !tree.base || !leaf_ids || !leaf_cnt || leaf_cap < 1 ||
      !ws.base || !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if (tree.bytes < zha_tree_bytes(g)) return ZHA_ERR_CAPACITY;
  if ((s = check_ws(g, nq, ZHA_OP_ROUTE, ws)) != ZHA_OK) return s;
  RouteCall c{g, nq, Q, q_pos, 0, p, tree.base, leaf_ids, leaf_cnt, leaf_cap, level_cnt, level_ids,
              (char*)ws.base, dev_status, (cudaStream_t)stream};
  return from_cuda(route_all(c));
}

zha_status zha_route_schedule(const zha_geom* g, const void* Q, const int64_t* q_pos, int32_t nq,
                              const double* p_levels, zha_buf tree, int32_t* leaf_ids,
                              int32_t* leaf_cnt, int32_t leaf_cap, int32_t* level_cnt,
                              int32_t* level_ids, zha_buf ws, int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!p_levels) return ZHA_ERR_INVALID_ARG;
  for (int l = 0; l < g->depth; ++l)
    if (!valid_p(p_levels[l])) return ZHA_ERR_INVALID_ARG;
  if (!Q || !q_pos || nq < 1 || !tree.base || !leaf_ids || !leaf_cnt || leaf_cap < 1 || !ws.base ||
      !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if (tree.bytes < zha_tree_bytes(g)) return ZHA_ERR_CAPACITY;
  if ((s = check_ws(g, nq, ZHA_OP_ROUTE, ws)) != ZHA_OK) return s;
  RouteCall c{g, nq, Q, q_pos, 0, p_levels[0], tree.base, leaf_ids, leaf_cnt, leaf_cap, level_cnt,
              level_ids, (char*)ws.base, dev_status, (cudaStream_t)stream, p_levels};
  return from_cuda(route_all(c));
}

zha_status zha_route_topk(const zha_geom* g, const void* Q, const int64_t* q_pos, int32_t nq,
                          const int32_t* k_levels, zha_buf tree, int32_t* leaf_ids, int32_t* leaf_cnt,
                          int32_t leaf_cap, int32_t* level_cnt, int32_t* level_ids, zha_buf ws,
                          int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!k_levels) return ZHA_ERR_INVALID_ARG;
  for (int l = 0; l < g->depth; ++l)
    if (k_levels[l] < 1) return ZHA_ERR_INVALID_ARG;
  if (!Q || !q_pos || nq < 1 || !tree.base || !leaf_ids || !leaf_cnt || leaf_cap < 1 || !ws.base ||
      !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if (tree.bytes < zha_tree_bytes(g)) return ZHA_ERR_CAPACITY;
  if ((s = check_ws(g, nq, ZHA_OP_ROUTE, ws)) != ZHA_OK) return s;
  RouteCall c{g, nq, Q, q_pos, 0, 1.0, tree.base, leaf_ids, leaf_cnt, leaf_cap, level_cnt, level_ids,
              (char*)ws.base, dev_status, (cudaStream_t)stream, nullptr, k_levels};
  return from_cuda(route_all(c));
}

zha_status zha_sparse_attn(const zha_geom* g, const void* Q, const void* K, const void* V,
                           const int64_t* q_pos, int32_t nq, const int32_t* leaf_ids,
                           const int32_t* leaf_cnt, int32_t leaf_cap, void* O, float* lse,
                           zha_buf ws, int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!Q || !K || !V || !q_pos || nq < 1 || !leaf_ids || !leaf_cnt || leaf_cap < 1 || !O ||
      !ws.base || !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if ((s = check_ws(g, nq, ZHA_OP_ATTN, ws)) != ZHA_OK) return s;
  AttnCall c{g, nq, Q, K, V, q_pos, 0, 0, leaf_ids, leaf_cnt, leaf_cap, O, lse, (char*)ws.base,
             dev_status, (cudaStream_t)stream};
  return from_cuda(attention(c));
}

zha_status zha_decode(const zha_geom* g, const void* q, const void* k_new, const void* v_new,
                      void* K, void* V, int64_t T, const float* qref, double p, zha_buf tree,
                      int32_t* leaf_ids, int32_t* leaf_cnt, int32_t leaf_cap, void* O,
                      zha_buf ws, int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!q || !k_new || !v_new || !K || !V || !qref || !valid_p(p) || !tree.base || !leaf_ids ||
      !leaf_cnt || leaf_cap < 1 || !O || !ws.base || !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if (T < 0 || T + 1 > g->t_cap) return ZHA_ERR_INVALID_ARG;
  if (tree.bytes < zha_tree_bytes(g)) return ZHA_ERR_CAPACITY;
  if ((s = check_ws(g, 1, ZHA_OP_DECODE, ws)) != ZHA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = append_tokens(*g, K, V, k_new, v_new, T, 1, st);
  if (e == cudaSuccess) e = tree_extend(*g, K, qref, tree.base, T, T + 1, st);
  if (e != cudaSuccess) return ZHA_ERR_CUDA;
  RouteCall rc{g, 1, q, nullptr, T, p, tree.base, leaf_ids, leaf_cnt, leaf_cap, nullptr, nullptr,
               (char*)ws.base, dev_status, st};
  if ((e = route_all(rc)) != cudaSuccess) return ZHA_ERR_CUDA;
  AttnCall ac{g, 1, q, K, V, nullptr, T, 0, leaf_ids, leaf_cnt, leaf_cap, O, nullptr,
              (char*)ws.base, dev_status, st};
  return from_cuda(attention(ac));
}

zha_status zha_prefill_attn(const zha_geom* g, const void* Q, const void* K, const void* V,
                            const int64_t* q_pos, int32_t nq, const int32_t* leaf_ids,
                            const int32_t* leaf_cnt, int32_t leaf_cap, void* O, float* lse,
                            zha_buf ws, int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (g->dtype != ZHA_BF16) return ZHA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !q_pos || nq < 1 || !leaf_ids || !leaf_cnt || leaf_cap < 1 || !O ||
      !ws.base || !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if ((s = check_ws(g, nq, ZHA_OP_PREFILL, ws)) != ZHA_OK) return s;
  PrefillCall c{g, nq, Q, K, V, q_pos, leaf_ids, leaf_cnt, leaf_cap, O, lse, (char*)ws.base, dev_status,
                (cudaStream_t)stream};
  return from_cuda(prefill_attention(c));
}

zha_status zha_check_bounded_wait(int64_t polls, int32_t* dev_status, int64_t* out, void* stream) {
  if (polls < 1 || polls > ((int64_t)1 << 32) || !dev_status || !out) return ZHA_ERR_INVALID_ARG;
  wait_check_launch((long long)polls, dev_status, (long long*)out, (cudaStream_t)stream);
  count_launch();
  return from_cuda(launch_status("wait_check_kernel"));
}

zha_status zha_dense_decode(const zha_geom* g, const void* Q, const void* K, const void* V,
                            const int64_t* q_pos, int32_t nq, void* O, float* lse, zha_buf ws,
                            int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!Q || !K || !V || !q_pos || nq < 1 || !O || !ws.base || !dev_status) return ZHA_ERR_INVALID_ARG;
  if ((s = check_ws(g, nq, ZHA_OP_DENSE, ws)) != ZHA_OK) return s;
  AttnCall c{g, nq, Q, K, V, q_pos, 0, 1, nullptr, nullptr, 1, O, lse, (char*)ws.base, dev_status,
             (cudaStream_t)stream};
  return from_cuda(attention(c));
}

zha_status zha_flat_index(const zha_geom* g, const void* Q, const void* K, const void* V,
                          const int64_t* q_pos, int32_t nq, double p, int32_t* leaf_ids,
                          int32_t* leaf_cnt, int32_t leaf_cap, void* O, zha_buf ws,
                          int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!Q || !K || !V || !q_pos || nq < 1 || !valid_p(p) || !leaf_ids || !leaf_cnt || leaf_cap < 1 ||
      !O || !ws.base || !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if ((s = check_ws(g, nq, ZHA_OP_FLAT, ws)) != ZHA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  RouteCall rc{g, nq, Q, q_pos, 0, p, const_cast<void*>(K), leaf_ids, leaf_cnt, leaf_cap, nullptr,
               nullptr, (char*)ws.base, dev_status, st};
  cudaError_t e = flat_select(rc);
  if (e != cudaSuccess) return ZHA_ERR_CUDA;
  AttnCall ac{g, nq, Q, K, V, q_pos, 0, 0, leaf_ids, leaf_cnt, leaf_cap, O, nullptr, (char*)ws.base,
              dev_status, st};
  return from_cuda(attention(ac));
}

}  // extern "C"
