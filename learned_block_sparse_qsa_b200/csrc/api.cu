// C-ABI of libqsa (declared in include/qsa.h): argument validation, geometry, dispatch.
// Every entry point validates its host-visible arguments synchronously, then enqueues kernels on
// the caller's stream.  Nothing here allocates device memory or synchronises.
#include <math.h>
#include <stdio.h>

#include "../../include/qsa.h"
#include "internal.h"

namespace qsa {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  if (dev < 64) cached[dev] = n;
  return n;
}

}  // namespace qsa

using qsa::Geometry;

namespace {

bool pow2_le(int x, int maxv) { return x >= 1 && x <= maxv && (x & (x - 1)) == 0; }

// Checks shared by every entry point; fills the geometry.
qsa_status_t make_geometry(const qsa_config_t* cfg, const qsa_batch_t* b, Geometry* g,
                           bool need_rows) {
  if (!cfg || !b) return QSA_ERR_INVALID_ARG;
  if (b->batch < 1 || b->num_q < 0 || b->max_pages_per_seq < 1 || b->num_pages < 1 ||
      b->max_pos < 0)
    return QSA_ERR_INVALID_ARG;
  if (!b->page_table || !b->err_flag) return QSA_ERR_INVALID_ARG;
  if (need_rows && b->num_q > 0 && (!b->q_seq || !b->q_pos)) return QSA_ERR_INVALID_ARG;
  if (cfg->block_tokens != 4 || cfg->page_tokens != 64 || cfg->idx_heads != 4)
    return QSA_ERR_UNSUPPORTED;
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return QSA_ERR_UNSUPPORTED;
  if (cfg->idx_dim != 32 && cfg->idx_dim != 64 && cfg->idx_dim != 128) return QSA_ERR_UNSUPPORTED;
  if (!pow2_le(cfg->num_kv_heads, 8)) return QSA_ERR_UNSUPPORTED;
  if (cfg->num_q_heads < cfg->num_kv_heads || cfg->num_q_heads % cfg->num_kv_heads != 0)
    return QSA_ERR_INVALID_ARG;
  if (!pow2_le(cfg->num_q_heads / cfg->num_kv_heads, 16)) return QSA_ERR_UNSUPPORTED;
  if (cfg->topk_blocks < 1 || cfg->topk_blocks > 512) return QSA_ERR_UNSUPPORTED;
  if (cfg->score_path < 0 || cfg->score_path > 5) return QSA_ERR_INVALID_ARG;
  if ((long long)b->max_pages_per_seq * 64 > (1LL << 30)) return QSA_ERR_UNSUPPORTED;
  g->Hq = cfg->num_q_heads;
  g->Hkv = cfg->num_kv_heads;
  g->D = cfg->head_dim;
  g->G = g->Hq / g->Hkv;
  g->Di = cfg->idx_dim;
  g->topk = cfg->topk_blocks;
  g->batch = b->batch;
  g->num_q = b->num_q;
  g->max_pages = b->max_pages_per_seq;
  g->num_pages = b->num_pages;
  g->max_pos = b->max_pos;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / sqrtf((float)g->D);
  g->scale_log2 = scale * 1.4426950408889634f;
  g->q_seq = b->q_seq;
  g->q_pos = b->q_pos;
  g->page_table = b->page_table;
  g->err = b->err_flag;
  return QSA_OK;
}

qsa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA; }

}  // namespace

extern "C" {

const char* qsa_status_string(qsa_status_t s) {
  switch (s) {
    case QSA_OK: return "ok";
    case QSA_ERR_INVALID_ARG: return "invalid argument";
    case QSA_ERR_UNSUPPORTED: return "unsupported shape";
    case QSA_ERR_WORKSPACE: return "workspace missing or too small";
    case QSA_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

int32_t qsa_version(void) { return 100; }

qsa_status_t qsa_workspace_size(const qsa_config_t* cfg, const qsa_batch_t* batch, qsa_op_t op,
                                int32_t num_splits, size_t* bytes) {
  if (!bytes) return QSA_ERR_INVALID_ARG;
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, false);
  if (st != QSA_OK) return st;
  switch (op) {
    case QSA_OP_INDEX_SCORE_TOPK:
      *bytes = qsa::score_workspace_bytes(g, qsa::resolve_score_path(g, cfg->score_path));
      return QSA_OK;
    case QSA_OP_SPARSE_ATTN_DECODE:
      *bytes = qsa::sparse_decode_workspace_bytes(g, qsa::resolve_sparse_splits(g, num_splits));
      return QSA_OK;
    case QSA_OP_DECODE_STEP:
      if (num_splits < 0) return QSA_ERR_INVALID_ARG;
      if (!qsa::decode_step_supported(g)) return QSA_ERR_UNSUPPORTED;
      *bytes = qsa::decode_step_workspace_bytes(g, num_splits);
      return QSA_OK;
    case QSA_OP_MERGE_CANDIDATES:
      if (num_splits < 1 || num_splits > qsa::kMaxCpParts) return QSA_ERR_INVALID_ARG;
      *bytes = qsa::cp_merge_workspace_bytes(g, num_splits);
      return QSA_OK;
    case QSA_OP_DENSE_ATTN_DECODE: {
      const int s = qsa::resolve_dense_splits(g, num_splits);
      *bytes = s > 1 ? qsa::dense_decode_workspace_bytes(g, s) : 0;
      return QSA_OK;
    }
    case QSA_OP_DISTILL_KL:
      *bytes = qsa::distill_tc_shape(g) ? qsa::distill_tc_workspace_bytes(g) : 0;
      return QSA_OK;
  }
  return QSA_ERR_INVALID_ARG;
}

qsa_status_t qsa_index_compress(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                const void* idx_k, const int32_t* new_seq,
                                const int32_t* new_pos, int32_t n_new, void* kcomp_pool,
                                qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, false);
  if (st != QSA_OK) return st;
  if (n_new < 0 || n_new % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (n_new == 0) return QSA_OK;
  if (!idx_k || !new_seq || !new_pos || !kcomp_pool) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx_k) | reinterpret_cast<uintptr_t>(kcomp_pool)) & 15)
    return QSA_ERR_INVALID_ARG;
  return from_cuda(qsa::launch_compress(g, idx_k, new_seq, new_pos, n_new, kcomp_pool,
                                        (cudaStream_t)stream));
}

qsa_status_t qsa_index_score_topk(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                  const void* idx_q, const void* idx_w, const void* kcomp_pool,
                                  int32_t* sel, int32_t* n_sel, float* sel_scores,
                                  void* workspace, size_t ws_bytes, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, true);
  if (st != QSA_OK) return st;
  if (g.num_q == 0) return QSA_OK;
  if (!idx_q || !idx_w || !kcomp_pool || !sel || !n_sel) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx_q) | reinterpret_cast<uintptr_t>(kcomp_pool)) & 15)
    return QSA_ERR_INVALID_ARG;
  const int path = qsa::resolve_score_path(g, cfg->score_path);
  const size_t need = qsa::score_workspace_bytes(g, path);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return QSA_ERR_WORKSPACE;
  if (!qsa::score_path_runnable(g, path)) return QSA_ERR_UNSUPPORTED;
  return from_cuda(qsa::launch_score_topk(g, path, idx_q, idx_w, kcomp_pool, sel, n_sel,
                                          sel_scores, workspace, ws_bytes, (cudaStream_t)stream));
}

qsa_status_t qsa_index_score_redo_flags(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                        void* workspace, size_t ws_bytes, int32_t** flags) {
  if (!flags) return QSA_ERR_INVALID_ARG;
  *flags = nullptr;
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, false);
  if (st != QSA_OK) return st;
  const int path = qsa::resolve_score_path(g, cfg->score_path);
  if (!workspace || ws_bytes < qsa::score_workspace_bytes(g, path)) return QSA_ERR_WORKSPACE;
  size_t off = 0;
  if (g.num_q > 0 && qsa::score_redo_offset(g, path, &off))
    *flags = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + off);
  return QSA_OK;
}

qsa_status_t qsa_index_scores(const qsa_config_t* cfg, const qsa_batch_t* batch,
                              const void* idx_q, const void* idx_w, const void* kcomp_pool,
                              float* scores, int64_t ld, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, true);
  if (st != QSA_OK) return st;
  if (g.num_q == 0) return QSA_OK;
  if (!idx_q || !idx_w || !kcomp_pool || !scores) return QSA_ERR_INVALID_ARG;
  if (ld < g.max_pos / 4) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx_q) | reinterpret_cast<uintptr_t>(kcomp_pool)) & 15)
    return QSA_ERR_INVALID_ARG;
  return from_cuda(qsa::launch_scores_only(g, idx_q, idx_w, kcomp_pool, scores, ld,
                                           (cudaStream_t)stream));
}

static qsa_status_t sparse_common(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                  const void* q, const void* k_pool, const void* v_pool,
                                  const int32_t* sel, const int32_t* n_sel, void* out,
                                  Geometry* g) {
  qsa_status_t st = make_geometry(cfg, batch, g, true);
  if (st != QSA_OK) return st;
  if (g->num_q == 0) return QSA_OK;
  if (!q || !k_pool || !v_pool || !sel || !n_sel || !out) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_pool) |
       reinterpret_cast<uintptr_t>(v_pool) | reinterpret_cast<uintptr_t>(out)) & 15)
    return QSA_ERR_INVALID_ARG;
  return QSA_OK;
}

qsa_status_t qsa_sparse_attn_prefill(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                     const void* q, const void* k_pool, const void* v_pool,
                                     const int32_t* sel, const int32_t* n_sel, void* out,
                                     float* lse, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = sparse_common(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, &g);
  if (st != QSA_OK || g.num_q == 0) return st;
  return from_cuda(qsa::launch_sparse_attn(g, q, k_pool, v_pool, sel, n_sel, g.topk + 1, out,
                                           lse, 1, nullptr, (cudaStream_t)stream));
}

qsa_status_t qsa_sparse_attn_decode(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                    const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* sel, const int32_t* n_sel, void* out,
                                    float* lse, int32_t num_splits, void* workspace,
                                    size_t ws_bytes, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = sparse_common(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, &g);
  if (st != QSA_OK || g.num_q == 0) return st;
  if (num_splits < 0) return QSA_ERR_INVALID_ARG;
  const int s = qsa::resolve_sparse_splits(g, num_splits);
  const size_t need = qsa::sparse_decode_workspace_bytes(g, s);
  if (need > 0 && (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)))
    return QSA_ERR_WORKSPACE;
  return from_cuda(qsa::launch_sparse_attn(g, q, k_pool, v_pool, sel, n_sel, g.topk + 1, out,
                                           lse, s, workspace, (cudaStream_t)stream));
}

qsa_status_t qsa_decode_step(const qsa_config_t* cfg, const qsa_batch_t* batch,
                             const void* idx_k_new, const int32_t* new_seq, const int32_t* new_pos,
                             int32_t n_new, void* kcomp_pool, const void* idx_q, const void* idx_w,
                             const void* q, const void* k_pool, const void* v_pool, int32_t* sel,
                             int32_t* n_sel, float* sel_scores, void* out, float* lse,
                             int32_t num_splits, void* workspace, size_t ws_bytes,
                             qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = sparse_common(cfg, batch, q, k_pool, v_pool, sel, n_sel, out, &g);
  if (st != QSA_OK || g.num_q == 0) return st;
  if (num_splits < 0 || n_new < 0 || n_new % 4 != 0) return QSA_ERR_INVALID_ARG;
  if (!idx_q || !idx_w || !kcomp_pool || (n_new > 0 && (!idx_k_new || !new_seq || !new_pos)))
    return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx_q) | reinterpret_cast<uintptr_t>(kcomp_pool) |
       reinterpret_cast<uintptr_t>(idx_k_new)) & 15)
    return QSA_ERR_INVALID_ARG;
  if (!qsa::decode_step_supported(g) || qsa::tmap_encode_fn_available() == 0) return QSA_ERR_UNSUPPORTED;
  const size_t need = qsa::decode_step_workspace_bytes(g, num_splits);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return QSA_ERR_WORKSPACE;
  return from_cuda(qsa::launch_decode_step(g, idx_k_new, new_seq, new_pos, n_new, kcomp_pool, idx_q,
                                           idx_w, q, k_pool, v_pool, sel, n_sel, sel_scores, out,
                                           lse, num_splits, workspace, (cudaStream_t)stream));
}

qsa_status_t qsa_cp_shard_positions(const int32_t* q_pos, int32_t num_q, int32_t shard_start,
                                    int32_t shard_len, int32_t* pos_sel, int32_t* pos_attn,
                                    qsa_stream_t stream) {
  if (num_q < 0 || shard_start < 0 || shard_len < 64 || shard_start % 64 || shard_len % 64)
    return QSA_ERR_INVALID_ARG;
  if (num_q == 0) return QSA_OK;
  if (!q_pos || !pos_sel || !pos_attn) return QSA_ERR_INVALID_ARG;
  return from_cuda(qsa::launch_cp_positions(q_pos, num_q, shard_start, shard_len, pos_sel, pos_attn,
                                            (cudaStream_t)stream));
}

qsa_status_t qsa_index_merge_candidates(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                        int32_t nparts, const int32_t* part_sel,
                                        const float* part_scores, const int32_t* part_block_lo,
                                        int32_t block_lo, int32_t block_hi, int32_t* sel,
                                        int32_t* n_sel, float* sel_scores, int32_t* local_sel,
                                        int32_t* local_n, void* workspace, size_t ws_bytes,
                                        qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, true);
  if (st != QSA_OK) return st;
  if (nparts < 1 || nparts > qsa::kMaxCpParts || !part_block_lo || block_lo < 0 || block_hi < block_lo)
    return QSA_ERR_INVALID_ARG;
  if (g.num_q == 0) return QSA_OK;
  if (!part_sel || !part_scores || !sel || !n_sel || !local_sel || !local_n) return QSA_ERR_INVALID_ARG;
  for (int p = 0; p < nparts; ++p)
    if (part_block_lo[p] < 0) return QSA_ERR_INVALID_ARG;
  const size_t need = qsa::cp_merge_workspace_bytes(g, nparts);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return QSA_ERR_WORKSPACE;
  return from_cuda(qsa::launch_cp_merge(g, nparts, part_sel, part_scores, part_block_lo, block_lo,
                                        block_hi, sel, n_sel, sel_scores, local_sel, local_n,
                                        workspace, (cudaStream_t)stream));
}

qsa_status_t qsa_attn_merge_partials(int32_t nparts, int32_t num_q, int32_t num_q_heads,
                                     int32_t head_dim, const void* part_out, const float* part_lse,
                                     void* out, float* lse, qsa_stream_t stream) {
  if (nparts < 1 || num_q < 0 || num_q_heads < 1 || (head_dim != 64 && head_dim != 128))
    return QSA_ERR_INVALID_ARG;
  if (num_q == 0) return QSA_OK;
  if (!part_out || !part_lse || !out) return QSA_ERR_INVALID_ARG;
  return from_cuda(qsa::launch_cp_merge_partials(nparts, num_q, num_q_heads, head_dim, part_out,
                                                 part_lse, out, lse, (cudaStream_t)stream));
}

qsa_status_t qsa_sparse_attn_backward(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                      const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* sel, const int32_t* n_sel, const void* out,
                                      const float* lse, const void* dout, float* dq,
                                      float* dk_pool, float* dv_pool, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = sparse_common(cfg, batch, q, k_pool, v_pool, sel, n_sel, const_cast<void*>(out), &g);
  if (st != QSA_OK || g.num_q == 0) return st;
  if (!lse || !dout || !dq || !dk_pool || !dv_pool) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(dout) | reinterpret_cast<uintptr_t>(dk_pool) |
       reinterpret_cast<uintptr_t>(dv_pool)) & 15)
    return QSA_ERR_INVALID_ARG;
  if (g.G > 8) return QSA_ERR_UNSUPPORTED;
  return from_cuda(qsa::launch_sparse_attn_bwd(g, q, k_pool, v_pool, sel, n_sel, out, lse, dout, dq,
                                               dk_pool, dv_pool, (cudaStream_t)stream));
}

qsa_status_t qsa_index_distill_kl(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                  const void* q, const void* k_pool, const void* idx_q,
                                  const void* idx_w, const void* kcomp_pool, float* kl, float* lse,
                                  float* teacher, int64_t ld, void* workspace, size_t ws_bytes,
                                  qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, true);
  if (st != QSA_OK || g.num_q == 0) return st;
  if (!q || !k_pool || !idx_q || !idx_w || !kcomp_pool || !kl) return QSA_ERR_INVALID_ARG;
  if (teacher && ld < g.max_pos / 4) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_pool) |
       reinterpret_cast<uintptr_t>(idx_q) | reinterpret_cast<uintptr_t>(kcomp_pool)) & 15)
    return QSA_ERR_INVALID_ARG;
  if (qsa::distill_tc_shape(g)) {  // the tensor-core form
    if (!qsa::tmap_encode_fn_available()) return QSA_ERR_UNSUPPORTED;
    if (!workspace || ws_bytes < qsa::distill_tc_workspace_bytes(g) ||
        (reinterpret_cast<uintptr_t>(workspace) & 15))
      return QSA_ERR_WORKSPACE;
    return from_cuda(qsa::launch_distill_tc(g, q, k_pool, idx_q, idx_w, kcomp_pool, kl, lse, teacher,
                                            ld, workspace, (cudaStream_t)stream));
  }
  return from_cuda(qsa::launch_distill(g, q, k_pool, idx_q, idx_w, kcomp_pool, kl, lse, teacher,
                                       ld, (cudaStream_t)stream));
}

qsa_status_t qsa_dense_attn_prefill(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                    const void* q, const void* k_pool, const void* v_pool,
                                    void* out, float* lse, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, true);
  if (st != QSA_OK || g.num_q == 0) return st;
  if (!q || !k_pool || !v_pool || !out) return QSA_ERR_INVALID_ARG;
  return from_cuda(qsa::launch_dense_attn(g, q, k_pool, v_pool, out, lse, 1, nullptr,
                                          (cudaStream_t)stream));
}

qsa_status_t qsa_dense_attn_decode(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                   const void* q, const void* k_pool, const void* v_pool,
                                   void* out, float* lse, int32_t num_splits, void* workspace,
                                   size_t ws_bytes, qsa_stream_t stream) {
  Geometry g;
  qsa_status_t st = make_geometry(cfg, batch, &g, true);
  if (st != QSA_OK || g.num_q == 0) return st;
  if (!q || !k_pool || !v_pool || !out || num_splits < 0) return QSA_ERR_INVALID_ARG;
  const int s = qsa::resolve_dense_splits(g, num_splits);
  if (s > 1) {
    const size_t need = qsa::dense_decode_workspace_bytes(g, s);
    if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
      return QSA_ERR_WORKSPACE;
  }
  return from_cuda(qsa::launch_dense_attn(g, q, k_pool, v_pool, out, lse, s, workspace,
                                          (cudaStream_t)stream));
}

}  // extern "C"
