/*
 * qsa_synth.h -- C-ABI of libqsa_synth.so, the seeded synthetic-input filler.
 *
 * This library belongs to the input generator, not to the attention method:
 * it writes counter-based pseudo-random bf16 values (SplitMix64 streams, see
 * qsa_synth/gen_core.h) into caller-owned device memory, so that benchmark
 * inputs of many GiB are created where they are used.  The numpy twin in
 * qsa_synth/__init__.py reproduces any element bit for bit on the host.
 *
 * Pointers are device pointers owned by the caller, except in the host fill;
 * `stream` is a cudaStream_t (NULL = legacy default stream).  Device calls are
 * asynchronous and return a cudaError_t value (0 = success) from the launch.
 */
#ifndef QSA_SYNTH_H
#define QSA_SYNTH_H
#include <stdint.h>
#ifdef __cplusplus
extern "C" {
#endif

/* Distribution codes. */
#define QSYN_DIST_NORMAL 0  /* Irwin-Hall(4) stand-in for N(0,1), bounded by +-3.46 */
#define QSYN_DIST_UNIFORM 1 /* U[0,1) on a 2^-24 grid */
#define QSYN_DIST_INT3 2    /* integers in [-3, 3] */

/* out: bf16 [n]; out[i] = value(seed, tid, offset + i). */
int qsyn_fill_linear(void* out, int64_t n, int64_t offset, uint64_t seed, uint64_t tid, int dist,
                     void* stream);

/* pool: bf16 [num_pages, page_tokens, row_elems].  page_owner: int32 [num_pages],
 * seq * max_pages + logical_page for a used page, -1 for a free page (zero-filled).
 * Element (page, slot, e) of a used page gets value(seed, tid,
 * (seq * seq_stride + logical_page * page_tokens + slot) * row_elems + e). */
int qsyn_fill_paged(void* pool, int64_t num_pages, int page_tokens, int row_elems,
                    const int32_t* page_owner, int max_pages, int64_t seq_stride, uint64_t seed,
                    uint64_t tid, int dist, void* stream);

/* Host memory: out bf16 [nrows, width]; row r holds value(seed, tid, starts[r] + e), e < width.
 * Runs on `threads` host threads (<= 0: all cores).  Returns 0, or 1 for a NULL pointer. */
int qsyn_fill_rows_host(void* out, const int64_t* starts, int64_t nrows, int64_t width,
                        uint64_t seed, uint64_t tid, int dist, int threads);

#ifdef __cplusplus
}
#endif
#endif
