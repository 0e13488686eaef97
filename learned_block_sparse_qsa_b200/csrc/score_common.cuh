// Pieces shared by the indexer scoring kernels (score.cu, score_tc.cu).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace qsa {

constexpr int kHi = 4;  // indexer query heads

struct ScoreArgs {
  const bf16* idx_q;  // [num_q, 4, DI]
  const bf16* idx_w;  // [num_q, 4]
  const bf16* kcomp;  // [num_pages, 16, DI]
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int num_q, batch, max_pages, num_pages, topk, max_pos;
  int32_t* sel;
  int32_t* n_sel;
  float* sel_scores;
  int sel_stride;
  int32_t* err;
};

// Swizzled byte offset of 16-byte chunk `c` of row `r` in a [rows][DI] bf16 shared tile, chosen
// so that ldmatrix over 8 consecutive rows touches 8 distinct bank groups.
template <int DI>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  if constexpr (DI >= 64) {
    return (uint32_t)(r * (DI * 2) + ((c ^ (r & 7)) << 4));
  } else {
    return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
  }
}

// Validate a query row; returns its block limit t/4 (number of candidates) or -1.
__device__ __forceinline__ int row_limit(const ScoreArgs& a, int r, int* seq_out) {
  const int seq = a.q_seq[r];
  const int pos = a.q_pos[r];
  if (seq < 0 || seq >= a.batch) {
    flag_error(a.err, QSA_DEVERR_SEQ);
    return -1;
  }
  if (pos < 0 || pos / 64 >= a.max_pages || pos > a.max_pos) {
    flag_error(a.err, QSA_DEVERR_POS);
    return -1;
  }
  *seq_out = seq;
  return pos / 4;
}

// cp.async one 64-block tile of sequence `seq`'s compressed keys into a swizzled [64][DI] tile.
template <int DI, int NTHREADS>
__device__ __forceinline__ void load_kcomp_tile(const ScoreArgs& a, int seq, int tile, int nb,
                                                uint32_t dst) {
  constexpr int CH = DI / 8;
  for (int i = threadIdx.x; i < 64 * CH; i += NTHREADS) {
    const int blk = i / CH, c = i % CH;
    const int b = tile * 64 + blk;
    bool valid = b < nb;
    const bf16* src = a.kcomp;
    if (valid) {
      const int page = a.page_table[(long long)seq * a.max_pages + (b >> 4)];
      if (page < 0 || page >= a.num_pages) {
        if (c == 0) flag_error(a.err, QSA_DEVERR_PAGE);
        valid = false;
      } else {
        src = a.kcomp + ((long long)page * 16 + (b & 15)) * DI + c * 8;
      }
    }
    cp_async16(dst + swz<DI>(blk, c), src, valid);
  }
}


inline ScoreArgs make_args(const Geometry& g, const void* idx_q, const void* idx_w, const void* kcomp,
                    int32_t* sel, int32_t* n_sel, float* sel_scores) {
  ScoreArgs a;
  a.idx_q = static_cast<const bf16*>(idx_q);
  a.idx_w = static_cast<const bf16*>(idx_w);
  a.kcomp = static_cast<const bf16*>(kcomp);
  a.q_seq = g.q_seq;
  a.q_pos = g.q_pos;
  a.page_table = g.page_table;
  a.num_q = g.num_q;
  a.batch = g.batch;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.topk = g.topk;
  a.max_pos = g.max_pos;
  a.sel = sel;
  a.n_sel = n_sel;
  a.sel_scores = sel_scores;
  a.sel_stride = g.topk + 1;
  a.err = g.err;
  return a;
}


// Tiled TMA loads (tensor map in kernel-parameter space) completing on an mbarrier.
__device__ __forceinline__ void tma2d(uint32_t dst, const CUtensorMap* m, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
      "l"((uint64_t)m), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
// The same load with an L2 eviction-priority policy (from l2_evict_first_policy below).
__device__ __forceinline__ void tma2d_hint(uint32_t dst, const CUtensorMap* m, int x, int y, uint64_t* bar,
                                           uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;\n" ::"r"(dst),
      "l"((uint64_t)m), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}
// Lines read once per call: first in line for eviction, so that the small tables read next
// (page table, selections) stay in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma3d(uint32_t dst, const CUtensorMap* m, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(dst),
      "l"((uint64_t)m), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}

// cuTensorMapEncodeTiled from the driver (looked up once), or nullptr.  In score_tc.cu.
PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn();

// score_tc.cu: the tcgen05 kernel (Di = 128) used by the streaming path.
// stream: the stream-K form (every SM) rather than one CTA per 128-row tile.
bool score_tc_stream_pays(const Geometry& g);
size_t score_tc_workspace_bytes(const Geometry& g, bool stream);
size_t score_tc_redo_offset(const Geometry& g, bool stream);  // byte offset of the redo flags [num_q]
cudaError_t launch_score_tc(const ScoreArgs& a, const Geometry& g, void* ws, int32_t** redo_out,
                            bool stream, cudaStream_t s);

// score_dec.cu: decode-sized batches (split warp lists + exact merge; Di = 128).
bool score_dec_plan_ok(const Geometry& g);        // the split-list plan fits (any driver)
size_t score_dec_workspace_bytes(const Geometry& g);
size_t score_dec_redo_offset(const Geometry& g);  // byte offset of the redo flags [num_q]
cudaError_t launch_score_dec(const ScoreArgs& a, const Geometry& g, void* ws, int32_t** redo_out,
                             cudaStream_t s);

}  // namespace qsa
