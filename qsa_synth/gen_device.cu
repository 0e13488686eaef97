// qsa_synth/gen_device.cu -- device-side fill of seeded synthetic inputs.
//
// Part of the input generator (not of the attention method): it writes the
// counter-based values defined in gen_core.h straight into device tensors so
// that multi-GiB KV pools never cross PCIe.  Values are indexed by LOGICAL
// coordinates (sequence, position, head, dim), never by physical placement, so
// the host can regenerate any element of a paged pool independently.
#include <cuda_runtime.h>
#include <stdint.h>
#include "gen_core.h"

namespace {

__global__ void fill_linear_kernel(uint16_t* __restrict__ out, int64_t n, int64_t offset,
                                   uint64_t key, int dist) {
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (; i < n; i += stride) out[i] = qsyn_value_bf16(qsyn_hash(key, (uint64_t)(offset + i)), dist);
}

// pool is [num_pages, page_tokens, row_elems]; page_owner[p] = seq * max_pages + logical
// page, or -1 for a free page (filled with zeros).  Logical element index is
// ((seq * seq_stride + pos) * row_elems + e) with pos = logical_page * page_tokens + slot.
__global__ void fill_paged_kernel(uint16_t* __restrict__ pool, int64_t num_pages, int page_tokens,
                                  int row_elems, const int32_t* __restrict__ page_owner,
                                  int max_pages, int64_t seq_stride, uint64_t key, int dist) {
  const int64_t page_elems = (int64_t)page_tokens * row_elems;
  const int64_t n = num_pages * page_elems;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (; i < n; i += stride) {
    const int64_t page = i / page_elems;
    const int64_t within = i - page * page_elems;
    const int owner = page_owner[page];
    uint16_t v = 0;
    if (owner >= 0) {
      const int64_t seq = owner / max_pages;
      const int64_t lp = owner - seq * max_pages;
      const int64_t slot = within / row_elems;
      const int64_t e = within - slot * row_elems;
      const int64_t pos = lp * page_tokens + slot;
      v = qsyn_value_bf16(qsyn_hash(key, (uint64_t)((seq * seq_stride + pos) * row_elems + e)), dist);
    }
    pool[i] = v;
  }
}

int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 64) g = 148 * 64;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" {

// out[i] = value(seed, tid, offset + i) for i < n.  Returns a cudaError_t code.
int qsyn_fill_linear(void* out, int64_t n, int64_t offset, uint64_t seed, uint64_t tid, int dist,
                     void* stream) {
  if (n <= 0) return 0;
  fill_linear_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)out, n, offset, qsyn_key(seed, tid), dist);
  return (int)cudaGetLastError();
}

int qsyn_fill_paged(void* pool, int64_t num_pages, int page_tokens, int row_elems,
                    const int32_t* page_owner, int max_pages, int64_t seq_stride, uint64_t seed,
                    uint64_t tid, int dist, void* stream) {
  if (num_pages <= 0) return 0;
  fill_paged_kernel<<<grid_for(num_pages * page_tokens * (int64_t)row_elems), 256, 0,
                      (cudaStream_t)stream>>>((uint16_t*)pool, num_pages, page_tokens, row_elems,
                                              page_owner, max_pages, seq_stride,
                                              qsyn_key(seed, tid), dist);
  return (int)cudaGetLastError();
}

}  // extern "C"
