// Context-parallel pieces of the layer: one sequence's context split across ranks, each rank
// holding the keys, values and compressed keys of one contiguous range of positions (a shard).
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token window
// with a selective view": the indexer keeps the best 512 micro-blocks of the whole context plus the
// tail block, and core attention runs over their positions.  Split by context:
//   1. every rank selects, exactly, the best candidates of its own shard (the layer's own scoring
//      and selection, run in the shard's local coordinates: qsa_cp_shard_positions);
//   2. the ranks' candidate lists are gathered; qsa_index_merge_candidates takes, per row, the best
//      512 of their union under the layer's order (score descending, lower block first) -- every
//      global winner is a winner of its own shard, so this equals the single-GPU selection -- and
//      also hands back the winners that live in this rank's shard, in local block ids;
//   3. every rank attends over its own winners (a partial output and its log-sum-exp), the
//      partials are gathered, and qsa_attn_merge_partials weights them by their log-sum-exp.
// The gathers are the callers' collectives (NCCL all-gather over NVLink between the steps).
#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace qsa {
namespace {

constexpr int CP_WARPS = 8;

__global__ void cp_positions_kernel(const int32_t* __restrict__ q_pos, int num_q, int start, int len,
                                    int32_t* __restrict__ pos_sel, int32_t* __restrict__ pos_attn) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= num_q) return;
  const int t = q_pos[i];
  // selection: candidates b < t/4 globally = local blocks below (t - start)/4, all of them when
  // the shard ends before t, none when it starts after t
  pos_sel[i] = t < start ? 0 : (t < start + len ? t - start : len);
  // attention: positions clipped at t; a shard wholly before t is attended in full
  pos_attn[i] = t < start ? 0 : (t < start + len ? t - start : len - 1);
}

struct MergeArgs {
  const int32_t* q_seq;
  const int32_t* q_pos;
  int num_q, batch, topk, nparts, stride;  // stride = topk + 1 (list length of every part)
  const int32_t* part_sel;                  // [nparts, num_q, stride] local block ids
  const float* part_scores;                 // [nparts, num_q, stride]
  int part_lo[kMaxCpParts];                 // first block of each part's shard
  int lo, hi;                               // this rank's blocks [lo, hi)
  int32_t* sel;
  int32_t* n_sel;
  float* sel_scores;
  int32_t* local_sel;
  int32_t* local_n;
  u64* buf;  // [num_q, nparts * stride] candidate keys
  int32_t* err;
};

// One warp per row: the union of the parts' candidates (their tails, marked +inf, and padding
// left out) as 64-bit keys, the need largest by the warp radix select, sorted by block; then the
// entries inside this rank's shard in local ids.
__global__ void __launch_bounds__(CP_WARPS * 32) merge_candidates_kernel(MergeArgs a) {
  __shared__ uint32_t hist[CP_WARPS][256];
  __shared__ uint32_t sblk[CP_WARPS][512];
  __shared__ float ssc[CP_WARPS][512];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * CP_WARPS + warp;
  if (row >= a.num_q) return;
  const int seq = a.q_seq[row], t = a.q_pos[row];
  if (seq < 0 || seq >= a.batch || t < 0) {
    flag_error(a.err, seq < 0 || seq >= a.batch ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);
    write_empty_selection(row, a.sel, a.n_sel, a.sel_scores, a.stride);
    for (int i = lane; i < a.stride; i += 32) a.local_sel[(long long)row * a.stride + i] = -1;
    if (lane == 0) a.local_n[row] = 0;
    return;
  }
  const int lim = t / 4;
  const int need = min(a.topk, lim);
  u64* buf = a.buf + (long long)row * a.nparts * a.stride;
  int cnt = 0;
  for (int p = 0; p < a.nparts; ++p) {
    const long long base = ((long long)p * a.num_q + row) * a.stride;
    for (int j0 = 0; j0 < a.stride; j0 += 32) {
      const int j = j0 + lane;
      bool keep = false;
      u64 key = 0;
      if (j < a.stride) {
        const int b = a.part_sel[base + j];
        const float s = a.part_scores[base + j];
        const int gb = b + a.part_lo[p];
        keep = b >= 0 && !(s != s) && s != __int_as_float(0x7f800000) && gb < lim;
        if (keep) key = make_key(s, (uint32_t)gb);
      }
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (keep) buf[cnt + __popc(bal & ((1u << lane) - 1u))] = key;
      cnt += __popc(bal);
    }
  }
  __syncwarp();
  int n = need;
  if (cnt < need) {  // a part sent fewer candidates than its shard holds: not a valid union
    flag_error(a.err, QSA_DEVERR_INTERNAL);
    n = cnt;
  }
  if (n > 0) warp_select_compact(buf, cnt, n, hist[warp]);
  __syncwarp();
  for (int i = lane; i < n; i += 32) {
    const u64 k = buf[i];
    sblk[warp][i] = key_block(k);
    ssc[warp][i] = key_score(k);
  }
  __syncwarp();
  if (n > 0) warp_sort_blocks(sblk[warp], ssc[warp], n);
  __syncwarp();
  write_selection(row, n, lim, sblk[warp], ssc[warp], a.sel, a.n_sel, a.sel_scores, a.stride);
  // this rank's share: the winners in [lo, hi) and the tail when it lies there, in local ids
  int w = 0;
  int32_t* lrow = a.local_sel + (long long)row * a.stride;
  for (int i0 = 0; i0 <= n; i0 += 32) {
    const int i = i0 + lane;
    const int b = i < n ? (int)sblk[warp][i] : (i == n ? lim : -1);
    const bool in = i <= n && b >= a.lo && b < a.hi;
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (in) lrow[w + __popc(bal & ((1u << lane) - 1u))] = b - a.lo;
    w += __popc(bal);
  }
  __syncwarp();
  for (int i = w + lane; i < a.stride; i += 32) lrow[i] = -1;
  if (lane == 0) a.local_n[row] = w;
}

// out[row][h] = sum_p exp(lse_p - L) o_p with L = log sum_p exp(lse_p): the partial attention
// outputs of the shards weighted by their share of the softmax normaliser.
__global__ void merge_partials_kernel(int nparts, int num_q, int Hq, int D,
                                      const bf16* __restrict__ part_out,
                                      const float* __restrict__ part_lse, bf16* __restrict__ out,
                                      float* lse) {
  const int row = blockIdx.x, h = blockIdx.y;
  float M = -INFINITY;
  for (int p = 0; p < nparts; ++p) M = fmaxf(M, part_lse[((long long)p * num_q + row) * Hq + h]);
  float L = 0.f;
  if (M != -INFINITY)
    for (int p = 0; p < nparts; ++p) {
      const float v = part_lse[((long long)p * num_q + row) * Hq + h];
      if (v != -INFINITY) L += expf(v - M);
    }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    if (L > 0.f)
      for (int p = 0; p < nparts; ++p) {
        const long long pi = ((long long)p * num_q + row) * Hq + h;
        const float v = part_lse[pi];
        if (v != -INFINITY) acc += expf(v - M) * __bfloat162float(part_out[pi * D + d]);
      }
    out[((long long)row * Hq + h) * D + d] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
  }
  if (lse && threadIdx.x == 0) lse[(long long)row * Hq + h] = L > 0.f ? M + logf(L) : -INFINITY;
}

}  // namespace

cudaError_t launch_cp_positions(const int32_t* q_pos, int num_q, int start, int len,
                                int32_t* pos_sel, int32_t* pos_attn, cudaStream_t s) {
  if (num_q == 0) return cudaSuccess;
  cp_positions_kernel<<<(num_q + 255) / 256, 256, 0, s>>>(q_pos, num_q, start, len, pos_sel, pos_attn);
  return cudaGetLastError();
}

size_t cp_merge_workspace_bytes(const Geometry& g, int nparts) {
  return (size_t)g.num_q * nparts * (g.topk + 1) * 8;
}

cudaError_t launch_cp_merge(const Geometry& g, int nparts, const int32_t* part_sel,
                            const float* part_scores, const int32_t* part_lo, int lo, int hi,
                            int32_t* sel, int32_t* n_sel, float* sel_scores, int32_t* local_sel,
                            int32_t* local_n, void* ws, cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  MergeArgs a;
  a.q_seq = g.q_seq;
  a.q_pos = g.q_pos;
  a.num_q = g.num_q;
  a.batch = g.batch;
  a.topk = g.topk;
  a.nparts = nparts;
  a.stride = g.topk + 1;
  a.part_sel = part_sel;
  a.part_scores = part_scores;
  for (int p = 0; p < kMaxCpParts; ++p) a.part_lo[p] = p < nparts ? part_lo[p] : 0;
  a.lo = lo;
  a.hi = hi;
  a.sel = sel;
  a.n_sel = n_sel;
  a.sel_scores = sel_scores;
  a.local_sel = local_sel;
  a.local_n = local_n;
  a.buf = static_cast<u64*>(ws);
  a.err = g.err;
  merge_candidates_kernel<<<(g.num_q + CP_WARPS - 1) / CP_WARPS, CP_WARPS * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_cp_merge_partials(int nparts, int num_q, int Hq, int D, const void* part_out,
                                     const float* part_lse, void* out, float* lse, cudaStream_t s) {
  if (num_q == 0) return cudaSuccess;
  merge_partials_kernel<<<dim3(num_q, Hq), D, 0, s>>>(nparts, num_q, Hq, D,
                                                      static_cast<const bf16*>(part_out), part_lse,
                                                      static_cast<bf16*>(out), lse);
  return cudaGetLastError();
}

}  // namespace qsa
