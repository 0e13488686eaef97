// qsa_sparse_attn_decode_noalloc: split-K sparse decode attention with library-owned scratch.
//
// Same computation and kernels as qsa_sparse_attn_decode, but the split-K partial results live
// in a fixed 4 MiB array in device global memory that belongs to this library, so the caller
// passes no workspace and nothing is allocated at call time.  It exists for callers that cannot
// allocate device memory when they run a step -- for example a serving engine whose memory
// planner owns every device allocation and forbids new ones after start-up, or a plugin host that
// gives plug-ins no allocator.
//
// The array is a file-scope __device__ variable, so every GPU that loads this library holds the
// 4 MiB until the process exits.  Host code cannot use the variable's name as a device address;
// the first call on each device (with that device current) looks the address up once with
// cudaGetSymbolAddress and caches it.  That first call therefore makes a synchronous runtime call
// and should come before any stream capture.  All calls share the array: calls that overlap on
// the GPU (different streams, or different host threads) race on it.  Nothing in it has to start
// at zero -- every partial the combine step reads is written earlier in the same call.  The
// per-device address cache itself is safe to fill from several host threads at once: each entry
// is atomic, and threads that race on a device's first call store the same address.
#include <atomic>

#include "../../include/qsa.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char qsa_decode_scratch[kScratchBytes];

std::atomic<void*> g_scratch_ptr[64];  // zero-initialised (static storage)

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, qsa_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" qsa_status_t qsa_sparse_attn_decode_noalloc(const qsa_config_t* cfg,
                                                      const qsa_batch_t* batch, const void* q,
                                                      const void* k_pool, const void* v_pool,
                                                      const int32_t* sel, const int32_t* n_sel,
                                                      void* out, float* lse, int32_t num_splits,
                                                      qsa_stream_t stream) {
  // Argument checks and the partials' size come from the workspace form (no launch, no allocation).
  size_t need = 0;
  qsa_status_t st = qsa_workspace_size(cfg, batch, QSA_OP_SPARSE_ATTN_DECODE, num_splits, &need);
  if (st != QSA_OK) return st;
  if (num_splits < 0) return QSA_ERR_INVALID_ARG;
  int32_t splits = num_splits;
  if (need > kScratchBytes) {
    if (num_splits > 0) return QSA_ERR_WORKSPACE;  // explicit split count does not fit in 4 MiB
    // automatic split count: the largest one whose partials fit (1 needs no scratch at all)
    int s = 64;
    for (; s > 1; --s) {
      size_t n = 0;
      if (qsa_workspace_size(cfg, batch, QSA_OP_SPARSE_ATTN_DECODE, s, &n) == QSA_OK && n <= kScratchBytes)
        break;
    }
    splits = s;
    qsa_workspace_size(cfg, batch, QSA_OP_SPARSE_ATTN_DECODE, splits, &need);
  }
  void* ws = nullptr;
  if (need > 0 && scratch_address(&ws) != cudaSuccess) return QSA_ERR_CUDA;
  return qsa_sparse_attn_decode(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, lse, splits, ws,
                                need, stream);
}
