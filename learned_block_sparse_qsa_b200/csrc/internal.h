// Internal launch interface between the C-ABI layer (api.cu) and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qsa.h"

namespace qsa {

struct Geometry {  // validated copy of the config + batch scalars
  int Hq, Hkv, D, G, Di, topk, batch, num_q, max_pages, num_pages, max_pos;
  float scale_log2;  // softmax scale * log2(e)
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int32_t* err;
};

int num_sms();

// compress.cu
cudaError_t launch_compress(const Geometry& g, const void* idx_k, const int32_t* new_seq,
                            const int32_t* new_pos, int n_new, void* kcomp, cudaStream_t s);

// score.cu
size_t score_workspace_bytes(const Geometry& g, int path);
int resolve_score_path(const Geometry& g, int requested);
bool score_path_runnable(const Geometry& g, int path);  // false: the driver lacks what it needs
int tmap_encode_fn_available();
bool score_redo_offset(const Geometry& g, int path, size_t* off);
cudaError_t launch_score_topk(const Geometry& g, int path, const void* idx_q, const void* idx_w,
                              const void* kcomp, int32_t* sel, int32_t* n_sel, float* sel_scores,
                              void* ws, size_t ws_bytes, cudaStream_t s);
cudaError_t launch_scores_only(const Geometry& g, const void* idx_q, const void* idx_w,
                               const void* kcomp, float* scores, int64_t ld, cudaStream_t s);

// score_dec.cu: the fused decode step (one cooperative launch)
bool decode_step_supported(const Geometry& g);
size_t decode_step_workspace_bytes(const Geometry& g, int num_splits);
cudaError_t launch_decode_step(const Geometry& g, const void* idx_k_new, const int32_t* new_seq,
                               const int32_t* new_pos, int n_new, void* kcomp, const void* idx_q,
                               const void* idx_w, const void* q, const void* k_pool,
                               const void* v_pool, int32_t* sel, int32_t* n_sel, float* sel_scores,
                               void* out, float* lse, int num_splits, void* ws, cudaStream_t s);

// attn.cu
int resolve_sparse_splits(const Geometry& g, int requested);
size_t sparse_decode_workspace_bytes(const Geometry& g, int splits);
cudaError_t launch_sparse_attn(const Geometry& g, const void* q, const void* k_pool,
                               const void* v_pool, const int32_t* sel, const int32_t* n_sel,
                               int sel_stride, void* out, float* lse, int splits, void* ws,
                               cudaStream_t s);

// dense.cu
int resolve_dense_splits(const Geometry& g, int requested);
// dense_tc.cu: the prefill form on tcgen05 (head_dim 128, 128 % G == 0, tensor maps available)
bool dense_tc_supported(const Geometry& g);
cudaError_t launch_dense_tc(const Geometry& g, const void* q, const void* k_pool, const void* v_pool,
                            void* out, float* lse, cudaStream_t s);
size_t dense_decode_workspace_bytes(const Geometry& g, int splits);
cudaError_t launch_dense_attn(const Geometry& g, const void* q, const void* k_pool,
                              const void* v_pool, void* out, float* lse, int splits, void* ws,
                              cudaStream_t s);

// cp.cu (context parallel)
constexpr int kMaxCpParts = 64;
cudaError_t launch_cp_positions(const int32_t* q_pos, int num_q, int start, int len,
                                int32_t* pos_sel, int32_t* pos_attn, cudaStream_t s);
size_t cp_merge_workspace_bytes(const Geometry& g, int nparts);
cudaError_t launch_cp_merge(const Geometry& g, int nparts, const int32_t* part_sel,
                            const float* part_scores, const int32_t* part_lo, int lo, int hi,
                            int32_t* sel, int32_t* n_sel, float* sel_scores, int32_t* local_sel,
                            int32_t* local_n, void* ws, cudaStream_t s);
cudaError_t launch_cp_merge_partials(int nparts, int num_q, int Hq, int D, const void* part_out,
                                     const float* part_lse, void* out, float* lse, cudaStream_t s);

// attn_bwd.cu
cudaError_t launch_sparse_attn_bwd(const Geometry& g, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* sel, const int32_t* n_sel,
                                   const void* out, const float* lse, const void* dout, float* dq,
                                   float* dk_pool, float* dv_pool, cudaStream_t s);

// distill.cu
// distill_tc.cu: the tensor-core form (head_dim 128, 8 query heads per KV head)
bool distill_tc_shape(const Geometry& g);
size_t distill_tc_workspace_bytes(const Geometry& g);
cudaError_t launch_distill_tc(const Geometry& g, const void* q, const void* k_pool, const void* idx_q,
                              const void* idx_w, const void* kcomp, float* kl, float* lse, float* teacher,
                              int64_t ld, void* ws, cudaStream_t s);
cudaError_t launch_distill(const Geometry& g, const void* q, const void* k_pool, const void* idx_q,
                           const void* idx_w, const void* kcomp, float* kl, float* lse,
                           float* teacher, int64_t ld, cudaStream_t s);

// combine (attn.cu): merge split partials [num_q, splits, Hq] of (o fp32 [D], lse2) -> bf16
cudaError_t launch_combine(const Geometry& g, const float* part_o, const float* part_lse,
                           int splits, void* out, float* lse, cudaStream_t s);

}  // namespace qsa
