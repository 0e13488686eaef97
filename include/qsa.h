/*
 * qsa.h -- C-ABI of libqsa, the B200 (sm_100a) Qwen Sparse Attention (QSA) layer.
 *
 * The layer, as described in the article "Qwen's million-token window has a 2,048-token
 * keyhole" (cronfeed.work), section "A million-token window with a selective view": an indexer
 * with four query heads and one shared key head averages its keys over 4-token micro-blocks,
 * scores the micro-blocks, keeps the best 512 (a 2,048-token budget that is the same at any
 * context length) together with the unfinished block at the tail of the sequence, maps them back
 * to token positions and runs the core attention there only.  Section "Three speed claims, three
 * different experiments" of the same article measures it against paged grouped-query attention
 * in chunked prefill and in multi-token decode; the dense entry points below are that baseline.
 *
 * Readings this library takes where the article is silent (all configurable fields excepted):
 *   k_b   = bf16_rne( (k[4b] + k[4b+1] + k[4b+2] + k[4b+3]) / 4 )   (computed exactly, then rounded)
 *   s_b(t) = sum_{h=0..3} w_h(t) * max(0, q_h(t) . k_b)                 (bf16 operands, fp32 accum.)
 *   candidates of query position t: blocks b < t / 4 (complete blocks not holding t);
 *   selection: top topk_blocks candidates by (score desc, block asc), plus the tail block t / 4;
 *   core attention of query head h uses key/value head h / (Hq / Hkv), softmax scale
 *   1/sqrt(head_dim) unless set, fp32 online softmax, bf16 output (round to nearest even).
 *
 * Memory model.  Every buffer is caller-owned device memory unless marked "host"; the library
 * allocates nothing and keeps no state beyond cached device attributes.  Every call is an
 * asynchronous launch on `stream` (a cudaStream_t; NULL = legacy default stream) and returns
 * after argument checks: QSA_OK, QSA_ERR_INVALID_ARG (bad sizes / NULL pointers / workspace too
 * small is QSA_ERR_WORKSPACE), QSA_ERR_UNSUPPORTED (shape outside what the kernels are built for),
 * or QSA_ERR_CUDA (a launch failed; cudaGetLastError() is cleared and folded into the status).
 * Problems that are only visible in device data (a page id outside the pool, a position outside
 * the page table, an out-of-range selection entry) never trap: the offending read is skipped or
 * zero-filled and a QSA_DEVERR_* bit is OR-ed into *batch->err_flag, which the caller zeroes and
 * reads after synchronising.
 *
 * Layouts (row-major, innermost last; bf16 = IEEE bfloat16 bit pattern):
 *   q          bf16 [num_q, Hq, D]            core-attention queries (post positional encoding)
 *   k_pool     bf16 [num_pages, 64, Hkv, D]   paged key cache; token p of sequence s lives in page
 *   v_pool     bf16 [num_pages, 64, Hkv, D]     page_table[s][p / 64], slot p % 64
 *   kcomp_pool bf16 [num_pages, 16, Di]       compressed indexer keys; block b of sequence s lives
 *                                             in page page_table[s][b / 16], slot b % 16
 *   idx_q      bf16 [num_q, 4, Di]            indexer queries;  idx_w bf16 [num_q, 4] head weights
 *   sel        int32 [num_q, topk+1]          selected blocks, ascending, tail block last, -1 pad
 *   n_sel      int32 [num_q]                  min(topk, t/4) + 1
 * q, k_pool, v_pool, kcomp_pool, idx_q, idx_k and the attention output must be 16-byte aligned
 * (QSA_ERR_INVALID_ARG otherwise).
 */
#ifndef QSA_H
#define QSA_H
#include <stddef.h>
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qsa_stream_t; /* same type as cudaStream_t */

typedef enum qsa_status {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,
  QSA_ERR_UNSUPPORTED = 2,
  QSA_ERR_WORKSPACE = 3,
  QSA_ERR_CUDA = 4
} qsa_status_t;

/* Bits OR-ed into *err_flag by the kernels. */
#define QSA_DEVERR_SEQ 1u      /* a sequence index outside [0, batch) */
#define QSA_DEVERR_POS 2u      /* a position < 0 or beyond the page table */
#define QSA_DEVERR_PAGE 4u     /* a page id outside [0, num_pages) */
#define QSA_DEVERR_GROUP 8u    /* compress: a 4-row group is not one aligned block of one sequence */
#define QSA_DEVERR_SEL 16u     /* attention: a selection entry outside [0, t/4] */
#define QSA_DEVERR_TIMEOUT 32u /* a bounded wait inside a kernel gave up */
#define QSA_DEVERR_INTERNAL 64u

typedef enum qsa_op {
  QSA_OP_INDEX_SCORE_TOPK = 1,
  QSA_OP_SPARSE_ATTN_DECODE = 2,
  QSA_OP_DENSE_ATTN_DECODE = 3,
  QSA_OP_MERGE_CANDIDATES = 4, /* num_splits = number of parts */
  QSA_OP_DECODE_STEP = 5,      /* num_splits as passed to qsa_decode_step */
  QSA_OP_DISTILL_KL = 6        /* qsa_index_distill_kl; num_splits unused */
} qsa_op_t;

typedef struct qsa_config {
  int32_t num_q_heads;  /* Hq, a multiple of num_kv_heads with Hq/Hkv in {1,2,4,8,16} */
  int32_t num_kv_heads; /* Hkv in {1, 2, 4, 8} */
  int32_t head_dim;     /* D in {64, 128} */
  int32_t idx_heads;    /* Hi, must be 4 */
  int32_t idx_dim;      /* Di in {32, 64, 128} */
  int32_t block_tokens; /* must be 4 */
  int32_t topk_blocks;  /* 1..512; the article's budget is 512 */
  int32_t page_tokens;  /* must be 64 */
  float softmax_scale;  /* <= 0 selects 1/sqrt(head_dim) */
  int32_t score_path;   /* qsa_index_score_topk algorithm, every one exact and equal:
                           0 auto: 3 for <= 128 rows when its plan fits, else 2 for <= 256 rows,
                             else 1, or 5 at idx_dim 128 when the rows' row tiles and the context
                             are such that spreading the work over every SM saves less than the
                             stream-K form's own costs (pure geometry);
                           1 many rows: at idx_dim 128 the tcgen05 tensor-core kernels in
                             their stream-K form (every SM takes an equal share of the (row tile,
                             key tile) work), whose unsettled rows the streaming kernel redoes;
                             else the streaming kernel;
                           2 materialised scores (any shape);
                           3 split lists for few rows (idx_dim 128; 2 when its plan does not fit);
                             the merge launch selects exactly over every candidate itself for a
                             row the lists cannot settle;
                           4 the mma.sync streaming kernel alone;
                           5 the tcgen05 kernel in its single-launch form, one CTA per 128-row
                             tile (idx_dim 128; 1 otherwise).
                           Paths 1, 3 and 5 at idx_dim 128 (and auto, which resolves to them) load
                           operands through tensor maps: when the driver offers no tensor-map
                           encoder, qsa_index_score_topk returns QSA_ERR_UNSUPPORTED rather than
                           switch kernels silently.  The resolution itself depends on the shape
                           only, so workspace sizes need no driver. */
} qsa_config_t;

typedef struct qsa_batch {
  int32_t batch;             /* host: number of sequences */
  int32_t num_q;             /* host: number of query rows */
  int32_t max_pages_per_seq; /* host: row length of page_table */
  int32_t num_pages;         /* host: pages in each pool */
  int32_t max_pos;           /* host: an upper bound on every q_pos (sizes grids/workspace) */
  const int32_t* q_seq;      /* device [num_q]: sequence of each query row */
  const int32_t* q_pos;      /* device [num_q]: absolute position t of each query row */
  const int32_t* page_table; /* device [batch, max_pages_per_seq]: physical page ids */
  int32_t* err_flag;         /* device [1]: QSA_DEVERR_* bits, zeroed by the caller */
} qsa_batch_t;

const char* qsa_status_string(qsa_status_t status);
int32_t qsa_version(void);

/* Bytes of workspace `op` needs for this batch (num_splits as passed to the call; 0 = auto).
 * *bytes is written on QSA_OK.  The workspace is caller-owned device memory, at least 256-byte
 * aligned, and may be reused between calls on the same stream. */
qsa_status_t qsa_workspace_size(const qsa_config_t* cfg, const qsa_batch_t* batch, qsa_op_t op,
                                int32_t num_splits, size_t* bytes);

/* Step (a), micro-block compression (article section "A million-token window with a selective
 * view": keys are compressed four tokens at a time).  The n_new rows of idx_k (bf16 [n_new, Di])
 * are the raw indexer keys of new tokens; n_new must be a multiple of 4 and rows 4j..4j+3 must
 * be positions 4b..4b+3 of one sequence (new_seq / new_pos: device int32 [n_new]).  For each such
 * group, kcomp_pool[page_table[s][b/16]][b%16] = bf16_rne(mean of the 4 rows), summed exactly.
 * A malformed group is skipped and flagged QSA_DEVERR_GROUP.  batch->q_seq/q_pos are unused. */
qsa_status_t qsa_index_compress(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                const void* idx_k, const int32_t* new_seq,
                                const int32_t* new_pos, int32_t n_new, void* kcomp_pool,
                                qsa_stream_t stream);

/* Steps (b)+(c), indexer scoring and selection (same section: the indexer ranks the
 * micro-blocks; a budget of 512 plus the unfinished tail block, per the article's opening).
 * For every query row: scores of all candidate blocks b < t/4 of its sequence (kcomp_pool must
 * hold them: compress runs first, including the blocks completed by this chunk), exact top
 * topk_blocks by (score desc, block asc), plus the tail block t/4; written ascending to
 * sel (int32 [num_q, topk+1], -1 padded), n_sel (int32 [num_q]) and, if not NULL, sel_scores
 * (float [num_q, topk+1]: the fp32 score of each selected block, +INFINITY for the tail, NaN
 * padding).  workspace: qsa_workspace_size(..., QSA_OP_INDEX_SCORE_TOPK, 0, ...) bytes. */
qsa_status_t qsa_index_score_topk(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                  const void* idx_q, const void* idx_w, const void* kcomp_pool,
                                  int32_t* sel, int32_t* n_sel, float* sel_scores,
                                  void* workspace, size_t ws_bytes, qsa_stream_t stream);

/* Diagnostic, no counterpart in the article.  Paths 1 (idx_dim 128), 3 and 5 first run a fast
 * kernel that settles most rows and flags the rest, which an exact selection then recomputes (the
 * exact streaming kernel; on path 3 the merge launch itself).
 * This host-only call returns in *flags the device address, inside `workspace`, of those flags
 * (int32 [num_q]: 1 = the row was recomputed, 0 = the fast kernel's own result) as the last
 * qsa_index_score_topk call with this config, batch shape and workspace left them; read them after
 * that call has completed.  *flags = NULL when the resolved path keeps no flags (paths 2 and 4,
 * path 1 below idx_dim 128, or an empty batch). */
qsa_status_t qsa_index_score_redo_flags(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                        void* workspace, size_t ws_bytes, int32_t** flags);

/* Diagnostic view of step (b): the fp32 score of every candidate block of every row, written to
 * scores (float [num_q, ld]); entries b >= t/4 are left untouched.  ld >= max_pos/4. */
qsa_status_t qsa_index_scores(const qsa_config_t* cfg, const qsa_batch_t* batch,
                              const void* idx_q, const void* idx_w, const void* kcomp_pool,
                              float* scores, int64_t ld, qsa_stream_t stream);

/* Steps (d)+(e), expansion and sparse core attention, prefill form (section "A million-token
 * window with a selective view": core attention only at the selected positions).  Row i attends
 * over positions {4b+j : b in sel[i][0..n_sel[i]), j < 4, 4b+j <= t} of its sequence, every query
 * head sharing the row's selection.  out: bf16 [num_q, Hq, D]; lse: float [num_q, Hq] natural-log
 * softmax normaliser, or NULL.  No workspace. */
qsa_status_t qsa_sparse_attn_prefill(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                     const void* q, const void* k_pool, const void* v_pool,
                                     const int32_t* sel, const int32_t* n_sel, void* out,
                                     float* lse, qsa_stream_t stream);

/* Same result as qsa_sparse_attn_prefill, computed split-K for few query rows (decode with
 * multi-token prediction, section "Three speed claims, three different experiments"): each row's
 * selected blocks are cut into num_splits pieces (0 = chosen from the device) processed in
 * parallel, then merged by their log-sum-exp (by the last piece of each row to finish, when
 * Hq/Hkv <= 8; else by a second kernel).  workspace: qsa_workspace_size(...,
 * QSA_OP_SPARSE_ATTN_DECODE, num_splits, ...) bytes; its contents need no initialisation. */
qsa_status_t qsa_sparse_attn_decode(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                    const void* q, const void* k_pool, const void* v_pool,
                                    const int32_t* sel, const int32_t* n_sel, void* out,
                                    float* lse, int32_t num_splits, void* workspace,
                                    size_t ws_bytes, qsa_stream_t stream);

/* The whole decode step in ONE launch (section "Three speed claims, three different experiments":
 * decode with batch 4 and three extra multi-token-prediction positions): compress the step's new
 * keys (as qsa_index_compress; n_new may be 0), select for every row (as qsa_index_score_topk),
 * and attend split-K (as qsa_sparse_attn_decode), in one cooperative kernel of one CTA per SM
 * whose CTAs wait for one another only on the data they need (bounded waits, ~1 s, then
 * QSA_DEVERR_TIMEOUT).  Results equal the three calls'.  Decode-sized batches: idx_dim 128,
 * Hq/Hkv <= 8, num_q <= 256 (QSA_ERR_UNSUPPORTED otherwise, or when the driver has no tensor-map
 * encoder).  workspace: qsa_workspace_size(..., QSA_OP_DECODE_STEP, num_splits, ...) bytes,
 * ZERO-FILLED before its first use: it holds the launch's synchronisation words, which every
 * completed call leaves at zero again (after a call that reported QSA_DEVERR_TIMEOUT, zero it
 * again).  Calls sharing a workspace must not overlap on the GPU. */
qsa_status_t qsa_decode_step(const qsa_config_t* cfg, const qsa_batch_t* batch,
                             const void* idx_k_new, const int32_t* new_seq, const int32_t* new_pos,
                             int32_t n_new, void* kcomp_pool, const void* idx_q, const void* idx_w,
                             const void* q, const void* k_pool, const void* v_pool, int32_t* sel,
                             int32_t* n_sel, float* sel_scores, void* out, float* lse,
                             int32_t num_splits, void* workspace, size_t ws_bytes,
                             qsa_stream_t stream);

/* No counterpart in the article: a variant of qsa_sparse_attn_decode for callers that cannot
 * allocate device memory at step time (for example a serving engine whose memory planner owns all
 * device memory and forbids allocations after start-up, or a plug-in host that gives plug-ins no
 * allocator).  Same arguments and results minus the workspace: the split-K partials live in a
 * 4 MiB array of device memory owned by libqsa (held by every GPU that loads the library until
 * the process exits).  num_splits > 0 whose partials (num_q * num_splits * Hq * (D + 1) floats)
 * exceed 4 MiB is rejected with QSA_ERR_WORKSPACE; num_splits = 0 picks the automatic split count,
 * lowered until the partials fit.  The first call on a device looks up the array's address (a
 * synchronous runtime call) and should come before any stream capture.  All calls share the
 * array: calls that overlap on the GPU race.  Nothing is allocated or freed. */
qsa_status_t qsa_sparse_attn_decode_noalloc(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                            const void* q, const void* k_pool, const void* v_pool,
                                            const int32_t* sel, const int32_t* n_sel, void* out,
                                            float* lse, int32_t num_splits, qsa_stream_t stream);

/* The comparison baseline (section "Three speed claims, three different experiments": paged
 * grouped-query attention): row i attends over every position 0..t of its sequence on the same
 * pools.  Rows of one sequence should be contiguous (they share key/value tiles).  Prefill form:
 * no workspace.  Decode form: split-K over the context with a log-sum-exp merge. */
qsa_status_t qsa_dense_attn_prefill(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                    const void* q, const void* k_pool, const void* v_pool,
                                    void* out, float* lse, qsa_stream_t stream);
qsa_status_t qsa_dense_attn_decode(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                   const void* q, const void* k_pool, const void* v_pool,
                                   void* out, float* lse, int32_t num_splits, void* workspace,
                                   size_t ws_bytes, qsa_stream_t stream);

/* ---- Context parallelism: one sequence's context split across ranks (not in the article, which
 * measures one accelerator; built so that a million-token context can be shared by several).
 * Rank r holds positions [start_r, start_r + len_r) of the sequence (multiples of 64: whole
 * pages) with a local page table of len_r/64 + 1 columns (the last one may name any valid page).
 * Per step: (1) qsa_cp_shard_positions gives each row's local positions; (2) the rank runs
 * qsa_index_score_topk with q_pos = pos_sel and its local tables: the exact best candidates of its
 * shard, in local block ids (its tail entry is ignored later); (3) the callers all-gather the ranks'
 * sel and sel_scores; (4) qsa_index_merge_candidates gives the global selection -- equal to the
 * single-accelerator one, because every global winner is a winner of its own shard -- and the
 * winners inside this rank's shard in local ids; (5) the rank attends over those with
 * q_pos = pos_attn (qsa_sparse_attn_prefill or _decode, lse requested); (6) the callers all-gather
 * the partial outputs and log-sum-exps and qsa_attn_merge_partials combines them. */

/* Local positions of the rows for the shard [shard_start, shard_start + shard_len) (device int32
 * [num_q] each): pos_sel = t - start clamped to [0, len] (len: every block of a shard that ends
 * before t is a candidate; 0: none of a shard that starts after t); pos_attn = t - start clamped
 * to [0, len - 1].  start and len: multiples of 64. */
qsa_status_t qsa_cp_shard_positions(const int32_t* q_pos, int32_t num_q, int32_t shard_start,
                                    int32_t shard_len, int32_t* pos_sel, int32_t* pos_attn,
                                    qsa_stream_t stream);

/* Exact merge of nparts candidate lists (section "A million-token window with a selective view":
 * the best 512 blocks of the whole context plus the tail).  part_sel / part_scores: device
 * [nparts, num_q, topk+1] as qsa_index_score_topk wrote them on each part (local block ids; +inf
 * scores mark tails and are skipped, -1 / NaN padding too); part_block_lo: HOST int32 [nparts], the
 * first global block of each part.  batch carries the GLOBAL q_seq / q_pos.  Writes the global
 * sel / n_sel / sel_scores (as qsa_index_score_topk would) and, for this rank's blocks
 * [block_lo, block_hi), local_sel (int32 [num_q, topk+1], local ids ascending, the tail included
 * when it lies there, -1 padded) and local_n (int32 [num_q]).  workspace:
 * qsa_workspace_size(..., QSA_OP_MERGE_CANDIDATES, nparts, ...) bytes.  nparts <= 64. */
qsa_status_t qsa_index_merge_candidates(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                        int32_t nparts, const int32_t* part_sel,
                                        const float* part_scores, const int32_t* part_block_lo,
                                        int32_t block_lo, int32_t block_hi, int32_t* sel,
                                        int32_t* n_sel, float* sel_scores, int32_t* local_sel,
                                        int32_t* local_n, void* workspace, size_t ws_bytes,
                                        qsa_stream_t stream);

/* out (bf16 [num_q, Hq, D]) and lse (float [num_q, Hq] or NULL) from nparts partial attentions
 * over disjoint position sets: part_out bf16 [nparts, num_q, Hq, D], part_lse float
 * [nparts, num_q, Hq] (natural log; -inf for an empty part): out = sum_p exp(lse_p - L) o_p with
 * L = log sum_p exp(lse_p). */
qsa_status_t qsa_attn_merge_partials(int32_t nparts, int32_t num_q, int32_t num_q_heads,
                                     int32_t head_dim, const void* part_out, const float* part_lse,
                                     void* out, float* lse, qsa_stream_t stream);

/* Backward of steps (d)+(e) with the selection held fixed (section "The indexer is trained, not
 * bolted on": after the dense warm-up the indexer and the backbone trained together through the
 * sparse layer; a top-k choice has no gradient).  Inputs as for qsa_sparse_attn_prefill plus the
 * forward's out (bf16 [num_q, Hq, D]) and lse (float [num_q, Hq], natural log) and the upstream
 * gradient dout (bf16 [num_q, Hq, D]).  Outputs: dq (float [num_q, Hq, D], written) and the
 * gradients of the key and value caches, dk_pool and dv_pool (float [num_pages, 64, Hkv, D], the
 * caches' layout in fp32): ADDED to, since every row that selected a block contributes to its
 * positions -- zero them first.  Hq/Hkv <= 8 (QSA_ERR_UNSUPPORTED otherwise).  No workspace. */
qsa_status_t qsa_sparse_attn_backward(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                      const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* sel, const int32_t* n_sel, const void* out,
                                      const float* lse, const void* dout, float* dq,
                                      float* dk_pool, float* dv_pool, qsa_stream_t stream);

/* The indexer's dense-distillation signal (section "The indexer is trained, not bolted on": the
 * indexer first learned from the full-attention distribution, token-level attention pooled into
 * blocks being the teacher).  For every query row at position t: the teacher is the dense causal
 * softmax attention of all Hq core heads over positions 0..t (softmax scale and head mapping as in
 * the core attention), summed over the 4 tokens of each candidate block b < t/4 and over the
 * heads, renormalised over the candidates; the student is the softmax over the same blocks of the
 * indexer scores s_b(t) (the selection scores); kl[i] (float [num_q]) = KL(teacher || student) in
 * nats, 0 when t < 4 and NaN for a row whose sequence or position is invalid (flagged).
 * Optional outputs: lse (float [num_q, Hq], natural-log normaliser of each head's dense softmax)
 * and teacher (float [num_q, ld], ld >= max_pos/4: the teacher distribution, entries b >= t/4
 * untouched).  Needs keys of positions 0..t in k_pool and the compressed keys of blocks < t/4;
 * reads no values.  A dense computation (two passes of q.k over the context).  At head_dim 128
 * with 8 query heads per KV head it runs on the tensor cores and needs a workspace of
 * qsa_workspace_size(..., QSA_OP_DISTILL_KL, 0, ...) bytes (block masses and indexer scores of
 * every row: 8 * num_q * (max_pos/4 + 1) bytes, rounded; QSA_ERR_WORKSPACE if smaller;
 * QSA_ERR_UNSUPPORTED when the driver has no tensor-map encoder); other shapes need none. */
qsa_status_t qsa_index_distill_kl(const qsa_config_t* cfg, const qsa_batch_t* batch,
                                  const void* q, const void* k_pool, const void* idx_q,
                                  const void* idx_w, const void* kcomp_pool, float* kl, float* lse,
                                  float* teacher, int64_t ld, void* workspace, size_t ws_bytes,
                                  qsa_stream_t stream);

/* No counterpart in the article: a self-test of failure detection.  Every pipelined kernel waits
 * on mbarriers with a bounded wait that, when it runs out, sets QSA_DEVERR_TIMEOUT in *err_flag
 * and lets the kernel return instead of hanging.  This call launches one CTA that waits, with that
 * same helper, on a phase that nothing completes, for limit_cycles (1e3..1e9 SM cycles; outside
 * that range QSA_ERR_INVALID_ARG): afterwards *err_flag has QSA_DEVERR_TIMEOUT set and the stream
 * and context remain usable. */
qsa_status_t qsa_selftest_wait_timeout(int32_t* err_flag, int64_t limit_cycles, qsa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
