// zha_sparse_attn_noalloc: the sparse attention of zha_sparse_attn for callers that can
// hand the library only their inputs and outputs and cannot give it a workspace.
//
// Some callers have no way to obtain extra device memory for a call: a plugin interface
// of an inference engine that passes only the operator's input and output buffers, or a
// process whose device memory is entirely reserved by another allocator, where a
// cudaMalloc would fail or would break the owner's accounting.  For them this entry point
// keeps its scratch (the union-of-heads staging lists, the work-item offsets and the
// split partials) in one file-scope device array of fixed size, ZHA_NOALLOC_SCRATCH_BYTES.
// The array is part of the loaded module: every GPU that loads the library holds it until
// the process exits.  The computation is the kernels of zha_sparse_attn; only the split
// size is chosen so that the scratch fits.
#include <mutex>

#include "zha_internal.cuh"

namespace zha {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ZHA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array, resolved once per device.  In host code the
// array's name is only a host-side stand-in for the symbol, so the address must come from
// cudaGetSymbolAddress with that device current.  The address is kept per device index
// for the life of the process: after a cudaDeviceReset the library must be reloaded.
constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

static cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();          // clear it, so that the next launch check reports its own error
      return e;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

// Smallest split size (chunks per work item, >= the default) whose layout fits the array;
// 0 if none does.
static int64_t fitting_cps(const zha_geom& g, int nq) {
  AttnWs w = attn_ws(g, nq, 0, 0);
  if (w.bytes <= (size_t)ZHA_NOALLOC_SCRATCH_BYTES) return w.cps;
  // one item per (unit, 4096-id block) is the fewest items (and the least scratch)
  const int64_t max_cps = kRange + 2;
  if (attn_ws(g, nq, 0, max_cps).bytes > (size_t)ZHA_NOALLOC_SCRATCH_BYTES) return 0;
  int64_t lo = w.cps, hi = max_cps;      // bytes shrink as cps grows
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) / 2;
    if (attn_ws(g, nq, 0, mid).bytes <= (size_t)ZHA_NOALLOC_SCRATCH_BYTES) hi = mid; else lo = mid;
  }
  return hi;
}

}  // namespace zha

using namespace zha;

extern "C" zha_status zha_sparse_attn_noalloc(const zha_geom* g, const void* Q, const void* K,
                                              const void* V, const int64_t* q_pos, int32_t nq,
                                              const int32_t* leaf_ids, const int32_t* leaf_cnt,
                                              int32_t leaf_cap, void* O, float* lse,
                                              int32_t* dev_status, void* stream) {
  zha_status s = zha_check_geom(g);
  if (s != ZHA_OK) return s;
  if (!Q || !K || !V || !q_pos || nq < 1 || !leaf_ids || !leaf_cnt || leaf_cap < 1 || !O ||
      !dev_status)
    return ZHA_ERR_INVALID_ARG;
  if (!call_fits(*g, nq)) return ZHA_ERR_UNSUPPORTED;
  const int64_t cps = fitting_cps(*g, nq);
  if (cps == 0) return ZHA_ERR_CAPACITY;
  void* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    note_cuda_error(e, "cudaGetSymbolAddress(noalloc scratch)");
    return ZHA_ERR_CUDA;
  }
  AttnCall c{g, nq, Q, K, V, q_pos, 0, 0, leaf_ids, leaf_cnt, leaf_cap, O, lse, (char*)scratch,
             dev_status, (cudaStream_t)stream, cps};
  return attention(c) == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA;
}
