// Step (a): micro-block compression of the shared indexer key head.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token
// window with a selective view": the indexer keys are compressed four tokens at a time.  This
// library's reading: the mean of the four raw keys, summed exactly (fp64 holds any sum of four
// bf16 values) and rounded once to bf16, nearest even.
//
// HBM-bound stream: each 16-byte load brings 8 dims of one raw key; 16 threads cover a 128-dim
// block, every warp reads 2 whole blocks (2 KiB) with fully coalesced 16-byte accesses and
// writes 512 contiguous bytes of the compressed pool.
#include "common.cuh"
#include "internal.h"

namespace qsa {
namespace {

template <int DI>
__global__ void __launch_bounds__(256) compress_kernel(
    const bf16* __restrict__ idx_k, const int32_t* __restrict__ new_seq,
    const int32_t* __restrict__ new_pos, int n_groups, const int32_t* __restrict__ page_table,
    int batch, int max_pages, int num_pages, bf16* __restrict__ kcomp, int32_t* err) {
  chain_wait();
  chain_release();
  constexpr int CH = DI / 8;  // 16-byte chunks per key row
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long grp = tid / CH;
  const int ch = (int)(tid % CH);
  if (grp >= n_groups) return;
  const long long r0 = grp * 4;
  // the four raw keys do not depend on the checks below: their loads go out first, so that
  // only the page-table read waits on the row metadata
  uint4 raw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) raw[i] = __ldg(reinterpret_cast<const uint4*>(idx_k + (r0 + i) * DI) + ch);
  const int seq = new_seq[r0];
  const int pos0 = new_pos[r0];
  bool ok = (pos0 >= 0) && (pos0 % 4 == 0);
#pragma unroll
  for (int i = 1; i < 4; ++i) ok = ok && new_seq[r0 + i] == seq && new_pos[r0 + i] == pos0 + i;
  if (!ok) {
    if (ch == 0) flag_error(err, QSA_DEVERR_GROUP);
    return;
  }
  if (seq < 0 || seq >= batch) {
    if (ch == 0) flag_error(err, QSA_DEVERR_SEQ);
    return;
  }
  const int lp = pos0 / 64;
  if (lp >= max_pages) {
    if (ch == 0) flag_error(err, QSA_DEVERR_POS);
    return;
  }
  const int page = page_table[(long long)seq * max_pages + lp];
  if (page < 0 || page >= num_pages) {
    if (ch == 0) flag_error(err, QSA_DEVERR_PAGE);
    return;
  }
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bf16* h = reinterpret_cast<const bf16*>(&raw[i]);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += (double)__bfloat162float(h[e]);
  }
  uint4 o;
  bf16* oh = reinterpret_cast<bf16*>(&o);
#pragma unroll
  for (int e = 0; e < 8; ++e) oh[e] = __double2bfloat16(acc[e] * 0.25);  // exact scale, one RNE
  const int slot = (pos0 / 4) % 16;
  reinterpret_cast<uint4*>(kcomp + ((long long)page * 16 + slot) * DI)[ch] = o;
}

}  // namespace

cudaError_t launch_compress(const Geometry& g, const void* idx_k, const int32_t* new_seq,
                            const int32_t* new_pos, int n_new, void* kcomp, cudaStream_t s) {
  const int n_groups = n_new / 4;
  if (n_groups == 0) return cudaSuccess;
  const long long threads = (long long)n_groups * (g.Di / 8);
  const int grid = (int)((threads + 255) / 256);
  auto* ik = static_cast<const bf16*>(idx_k);
  auto* kc = static_cast<bf16*>(kcomp);
  auto* kernel = g.Di == 32 ? compress_kernel<32> : g.Di == 64 ? compress_kernel<64> : compress_kernel<128>;
  return launch_chained(kernel, dim3(grid), dim3(256), 0, s, ik, new_seq, new_pos, n_groups, g.page_table, g.batch,
                        g.max_pages, g.num_pages, kc, g.err);
}

}  // namespace qsa
