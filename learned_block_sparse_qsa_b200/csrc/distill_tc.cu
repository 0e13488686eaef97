// The indexer's dense-distillation signal on the 5th-generation tensor cores (head_dim 128,
// 8 query heads per KV head): KL(teacher || indexer) per query row.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "The indexer is
// trained, not bolted on": before sparse training the indexer learned from the full-attention
// distribution, with token-level attention pooled into blocks as the teacher.  Readings (the
// article gives no formula): the teacher of query position t is the dense causal softmax
// attention of every core query head over positions 0..t, summed over the 4 tokens of each
// candidate block b < t/4 and over all query heads, renormalised over the candidates; the
// student is the softmax of the indexer's block scores over the same candidates; the loss is
// KL(teacher || student) in nats (0 for rows without candidates).
//
// Three launches:
//   distill_tc_kernel  CTA = two query tiles of 128 rows (16 tokens x the 8 query heads of one KV
//                      head each) sharing every K tile; two passes over the context with S = Q K^T
//                      in tensor memory (double-buffered per query tile).  Eight softmax warps per
//                      query tile: a warp reads 32 rows (its lane quarter) x 64 of the tile's 128
//                      columns.  Pass 1: each row's running maximum and sum in base 2 per column
//                      half, combined once through shared memory (the row's dense log-sum-exp).
//                      Pass 2: the probabilities 2^(scale s - lse), summed within each 4-position
//                      block, then over the 8 heads of the token by a shuffle reduce-scatter (each
//                      lane ends with 2 block sums), added into the block masses of the token in
//                      global memory (one 8-byte reduction per KV head and block pair).
//   scores             the indexer scores of every candidate (the materialised scoring kernel).
//   distill_finish     one CTA per row: M = sum m, A = sum m ln m, B = sum m s and the
//                      log-sum-exp of s over the candidates; KL = A/M - ln M - B/M + lse(s); the
//                      teacher m / M when asked for.
#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"
#include "tc_common.cuh"

namespace qsa {
namespace {

constexpr int DK_ROWS = 128;  // MMA M (one query tile)
constexpr int DK_NQ = 2;      // query tiles per CTA
constexpr int DK_G = 8;       // query heads per KV head of this layout
constexpr int DK_TQ = DK_ROWS / DK_G;
constexpr int DK_POS = 128;   // positions per K tile (N of S)
constexpr int DK_NST = 4;     // K stages
constexpr int DK_SMW = 8;     // softmax warps per query tile: 4 lane quarters x 2 column halves
constexpr int DK_COLS = DK_POS / 2;  // S columns per softmax warp
constexpr int DK_THREADS = (2 + DK_NQ * DK_SMW) * 32;
constexpr int DK_HALF = DK_ROWS * 128;   // one 64-column (128-byte) half of a 128-row tile
constexpr int DK_Q_BYTES = 2 * DK_HALF;  // query tile, K-major: [k-half][row][128 B]
constexpr int DK_K_BYTES = 2 * DK_HALF;  // K tile, K-major: [k-half][position][128 B]
constexpr uint32_t kIdescDK = idesc_bf16(DK_ROWS, DK_POS, false);

struct DkMisc {
  uint64_t qload, k_full[DK_NST], k_empty[DK_NST], s_full[DK_NQ][2], s_empty[DK_NQ][2], mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int issued, consumed;  // K tiles issued by the producer / waited for by the MMA issuer
  int seg, tmax, ntile;
  uint32_t done[1];   // tokens already handled (bit per token; 32 tokens per CTA)
  uint32_t inseg[1];  // tokens of the current segment
  float2 xch[DK_NQ][DK_ROWS][2];  // pass-1 (max, sum) of each row's two column halves
};
constexpr int DK_SMEM = DK_NQ * DK_Q_BYTES + DK_NST * DK_K_BYTES + (int)((sizeof(DkMisc) + 127) / 128 * 128);
static_assert(DK_SMEM <= 232448, "shared memory budget");
static_assert(DK_NQ * DK_TQ <= 32, "token bit masks");

struct DkArgs {
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int num_q, batch, max_pages, num_pages, max_pos, Hq;
  float scale_log2;
  float* lse;   // [num_q, Hq] or nullptr
  float* mass;  // [num_q, ldm], zeroed
  long long ldm;
  int32_t* err;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool dk_valid(const DkArgs& a, int r) {
  const int s = a.q_seq[r], t = a.q_pos[r];
  return s >= 0 && s < a.batch && t >= 0 && t <= a.max_pos && t / 64 < a.max_pages;
}

__global__ void __launch_bounds__(DK_THREADS, 1)
    distill_tc_kernel(DkArgs a, const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + DK_NQ * DK_Q_BYTES;
  DkMisc* m = reinterpret_cast<DkMisc*>(sK + DK_NST * DK_K_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NT = DK_NQ * DK_TQ;
  const int tok0 = blockIdx.x * NT;
  const int g = blockIdx.y;

  if (smem_addr(smem) & 1023) {  // operand tiles need 1024-byte alignment
    if (tid == 0) flag_error(a.err, QSA_DEVERR_INTERNAL);
    return;
  }
  if (tid == 0) {
    mbar_init(&m->qload, 1);
    for (int s = 0; s < DK_NST; ++s) {
      mbar_init(&m->k_full[s], 1);
      mbar_init(&m->k_empty[s], 1);
    }
    for (int q = 0; q < DK_NQ; ++q)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&m->s_full[q][b], 1);
        mbar_init(&m->s_empty[q][b], DK_SMW);
      }
    mbar_init(&m->mma_done, 1);
    m->abort_flag = 0;
    m->issued = 0;
    m->consumed = 0;
    uint32_t done = 0;  // rows past num_q and invalid rows (flagged) are done from the start
    for (int i = 0; i < NT; ++i) {
      const int r = tok0 + i;
      bool bad = r >= a.num_q;
      if (!bad && !dk_valid(a, r)) {
        const int s = a.q_seq[r];
        flag_error(a.err, (s < 0 || s >= a.batch) ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);
        bad = true;
      }
      if (bad) done |= 1u << i;
    }
    m->done[0] = done;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(
        smem_addr(&m->tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = m->tmem_base;

  if (warp == 0 && lane == 0) {  // the query tiles, once: rows past num_q read as zeros
    mbar_arrive_expect_tx(&m->qload, DK_NQ * DK_Q_BYTES);
    for (int q = 0; q < DK_NQ; ++q)
      for (int kh = 0; kh < 2; ++kh)
        tma3d(smem_addr(sQ + q * DK_Q_BYTES + kh * DK_HALF), &tmQ, kh * 64, g * DK_G, tok0 + q * DK_TQ,
              &m->qload);
  }

  const int qt = warp >= 2 ? (warp - 2) / DK_SMW : 0;
  const int half = warp >= 2 ? ((warp - 2) % DK_SMW) / 4 : 0;  // the warp's 64 of the tile's columns
  const int row = 32 * (warp & 3) + lane;
  const int tok = qt * DK_TQ + row / DK_G, head = row % DK_G;

  int gbase = 0;  // tiles of earlier segments, both passes (every role counts the same tiles)
  for (;;) {
    __syncthreads();
    if (tid == 0) {  // next segment: the sequence of the first token not yet done
      int seg = -1, tmax = -1;
      uint32_t in = 0;
      for (int i = 0; i < NT; ++i) {
        if ((m->done[0] >> i) & 1u) continue;
        const int s = a.q_seq[tok0 + i];
        if (seg < 0) seg = s;
        if (s == seg) {
          in |= 1u << i;
          tmax = max(tmax, a.q_pos[tok0 + i]);
        }
      }
      m->inseg[0] = in;
      m->seg = seg;
      m->tmax = tmax;
      m->ntile = seg < 0 ? 0 : tmax / DK_POS + 1;
    }
    __syncthreads();
    const int seg = m->seg;
    if (seg < 0 || m->abort_flag) break;
    const int ntile = m->ntile;
    const int L = 2 * ntile;  // pass 1 then pass 2

    if (warp == 0) {
      // ---------------------------------------------------------------- TMA producer
      if (lane == 0) {
        const int32_t* pt = a.page_table + (long long)seg * a.max_pages;
        for (int i = 0; i < L; ++i) {
          const int gj = gbase + i, s = gj % DK_NST, j = i % ntile;
          if (gj >= DK_NST && !mbar_wait(&m->k_empty[s], ((gj / DK_NST) & 1) ^ 1, a.err)) {
            m->abort_flag = 1;
            break;
          }
          int pid[2];
          for (int pg = 0; pg < 2; ++pg) {  // pages past the table hold only masked positions
            const int lp = 2 * j + pg;
            int p = 0;
            if (lp < a.max_pages) {
              p = pt[lp];
              if (p < 0 || p >= a.num_pages) {
                flag_error(a.err, QSA_DEVERR_PAGE);
                p = 0;
              }
            }
            pid[pg] = p;
          }
          uint8_t* st = sK + s * DK_K_BYTES;
          mbar_arrive_expect_tx(&m->k_full[s], DK_K_BYTES);
          for (int pg = 0; pg < 2; ++pg)
            for (int hh = 0; hh < 2; ++hh)  // [k-half hh][positions pg*64..][128 B]
              tma3d(smem_addr(st + hh * DK_HALF + pg * (DK_HALF / 2)), &tmK, hh * 64, g, pid[pg] * 64,
                    &m->k_full[s]);
          m->issued = gj + 1;
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        bool ok = gbase > 0 || mbar_wait(&m->qload, 0, a.err);
        for (int i = 0; ok && i < L; ++i) {
          const int gj = gbase + i, s = gj % DK_NST, b = gj & 1;
          if (!mbar_wait(&m->k_full[s], (gj / DK_NST) & 1, a.err)) { ok = false; break; }
          m->consumed = gj + 1;
          const uint32_t kb = smem_addr(sK + s * DK_K_BYTES);
          for (int q = 0; ok && q < DK_NQ; ++q) {
            if (gj >= 2 && !mbar_wait(&m->s_empty[q][b], ((gj >> 1) & 1) ^ 1, a.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t qa = smem_addr(sQ + q * DK_Q_BYTES);
#pragma unroll
            for (int ks = 0; ks < 128 / 16; ++ks) {
              const uint64_t ad = sw128_desc(qa + (ks >> 2) * DK_HALF + (ks & 3) * 32);
              const uint64_t bd = sw128_desc(kb + (ks >> 2) * DK_HALF + (ks & 3) * 32);
              umma_bf16(tbase + q * 256 + b * 128, ad, bd, kIdescDK, ks > 0 ? 1u : 0u);
            }
            umma_commit(&m->s_full[q][b]);
          }
          if (ok) umma_commit(&m->k_empty[s]);
        }
        if (!ok) m->abort_flag = 1;
      }
    } else {
      // ---------------------------------------------------------------- softmax + pooling
      const bool act = (m->inseg[0] >> tok) & 1u;
      const int t = act ? a.q_pos[tok0 + tok] : -1;
      const int nb = t >> 2;  // candidate blocks b < t/4 (t = -1: none)
      const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
      float mx = -INFINITY, sum = 0.f, lse2 = -INFINITY;
      bool dead = false;
      for (int i = 0; i < L; ++i) {
        const int gj = gbase + i, b = gj & 1, j = i % ntile, P0 = j * DK_POS + half * DK_COLS;
        const bool pass2 = i >= ntile;
        if (!dead) {
          const bool okw = mbar_wait(&m->s_full[qt][b], (gj >> 1) & 1, a.err);
          if (__any_sync(0xffffffffu, !okw)) {
            m->abort_flag = 1;
            dead = true;
          }
        }
        float v[DK_COLS];
        if (!dead) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < DK_COLS / 16; ++c) {
            float x[16];
            tmem_ld16(tbase + lb + qt * 256 + b * 128 + half * DK_COLS + c * 16, x);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[c * 16 + e] = x[e];
          }
          tmem_wait_ld();
          tc_fence_before();
        } else {
#pragma unroll
          for (int c = 0; c < DK_COLS; ++c) v[c] = -INFINITY;
        }
        __syncwarp();
        if (lane == 0 && !dead) mbar_arrive(&m->s_empty[qt][b]);
        if (P0 + DK_COLS - 1 > t) {  // mask positions after t
#pragma unroll
          for (int c = 0; c < DK_COLS; ++c) v[c] = P0 + c <= t ? v[c] : -INFINITY;
        }
        if (!pass2) {
          // pass 1: running maximum and sum of 2^(scale s) in base 2 over this half's columns
          float tm[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) tm[e] = v[e];
#pragma unroll
          for (int c = 8; c < DK_COLS; c += 8)
#pragma unroll
            for (int e = 0; e < 8; ++e) tm[e] = fmaxf(tm[e], v[c + e]);
          const float tmx = fmaxf(fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3])),
                                  fmaxf(fmaxf(tm[4], tm[5]), fmaxf(tm[6], tm[7]))) * a.scale_log2;
          const float mn = fmaxf(mx, tmx);
          if (mn != -INFINITY) {
            float ps[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) ps[e] = 0.f;
#pragma unroll
            for (int c = 0; c < DK_COLS; ++c) ps[c & 7] += fast_exp2(fmaf(v[c], a.scale_log2, -mn));
            const float ts = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
            sum = (mx == -INFINITY ? 0.f : sum * fast_exp2(mx - mn)) + ts;
            mx = mn;
          }
          if (i == ntile - 1) {  // both halves: the row's log-sum-exp, base 2
            m->xch[qt][row][half] = make_float2(mx, sum);
            named_bar_sync(1 + qt, DK_SMW * 32);
            const float2 o = m->xch[qt][row][half ^ 1];
            const float M2 = fmaxf(mx, o.x);
            const float S2 = (mx == -INFINITY ? 0.f : sum * fast_exp2(mx - M2)) +
                             (o.x == -INFINITY ? 0.f : o.y * fast_exp2(o.x - M2));
            lse2 = S2 > 0.f ? M2 + log2f(S2) : -INFINITY;
            if (act && a.lse && half == 0)  // natural log
              a.lse[(long long)(tok0 + tok) * a.Hq + g * DK_G + head] = lse2 * 0.69314718055994531f;
          }
        } else {
          // pass 2: block masses of this head's probabilities, then the 8 heads' sum
          const float nl = lse2 == -INFINITY ? -INFINITY : -lse2;
          float bs[DK_COLS / 4];
#pragma unroll
          for (int k = 0; k < DK_COLS / 4; ++k) {
            float s4 = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) s4 += fast_exp2(fmaf(v[4 * k + e], a.scale_log2, nl));
            bs[k] = s4;
          }
          // reduce-scatter over the token's 8 lanes: lane bits 2, 1, 0 pick halves of 8, 4, 2
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const bool up = lane & 4;
            const float keep = up ? bs[8 + k] : bs[k], give = up ? bs[k] : bs[8 + k];
            bs[k] = keep + __shfl_xor_sync(0xffffffffu, give, 4);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const bool up = lane & 2;
            const float keep = up ? bs[4 + k] : bs[k], give = up ? bs[k] : bs[4 + k];
            bs[k] = keep + __shfl_xor_sync(0xffffffffu, give, 2);
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const bool up = lane & 1;
            const float keep = up ? bs[2 + k] : bs[k], give = up ? bs[k] : bs[2 + k];
            bs[k] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
          }
          const int blk = P0 / 4 + ((lane >> 2) & 1) * 8 + ((lane >> 1) & 1) * 4 + (lane & 1) * 2;
          if (act && !dead && blk < nb) {  // blk is even: the pair is 8-byte aligned
            float* dst = a.mass + (long long)(tok0 + tok) * a.ldm + blk;
            if (blk + 1 < nb)
              atomicAdd(reinterpret_cast<float2*>(dst), make_float2(bs[0], bs[1]));
            else
              atomicAdd(dst, bs[0]);
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0) m->done[0] |= m->inseg[0];
    gbase += L;
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (m->abort_flag && warp == 0 && lane == 0) {  // let copies still in flight land first
    mbar_wait(&m->qload, 0, a.err);
    for (int gj = m->consumed; gj < m->issued; ++gj)
      mbar_wait(&m->k_full[gj % DK_NST], (gj / DK_NST) & 1, a.err);
  }
  if (warp == 1) {
    if (lane == 0 && gbase > 0) {  // every issued MMA has completed before TMEM is released
      umma_commit(&m->mma_done);
      mbar_wait(&m->mma_done, 0, a.err);
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tbase));
  }
}

// One 256-thread CTA per row: the KL from the block masses and the indexer scores of its
// candidates.  Two sweeps of the row: the largest score, then the sums (per-element logarithms and
// exponentials in fp32, each thread's sums in fp64, reduced over the CTA).
constexpr int DF_THREADS = 256;

__device__ __forceinline__ double df_block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();  // red[] may still be read by the previous reduction
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int w = 0; w < DF_THREADS / 32; ++w) t += red[w];
  return t;
}

__global__ void __launch_bounds__(DF_THREADS) distill_finish_kernel(DkArgs a, const float* __restrict__ scores,
                                                                   long long lds, float* __restrict__ kl,
                                                                   float* __restrict__ teacher, long long ldt) {
  __shared__ double red[DF_THREADS / 32];
  __shared__ float fred[DF_THREADS / 32];
  const int r = blockIdx.x, tid = threadIdx.x;
  if (!dk_valid(a, r)) {  // flagged by the first launch
    if (tid == 0) kl[r] = __int_as_float(0x7fc00000);
    return;
  }
  const int nb = a.q_pos[r] >> 2;
  const float* mrow = a.mass + (long long)r * a.ldm;
  const float* srow = scores + (long long)r * lds;
  float smax = -INFINITY;
  for (int b = tid; b < nb; b += DF_THREADS) smax = fmaxf(smax, srow[b]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
  if ((tid & 31) == 0) fred[tid >> 5] = smax;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < DF_THREADS / 32; ++w) smax = fmaxf(smax, fred[w]);
  double M = 0.0, A = 0.0, B = 0.0, Z = 0.0;
  for (int b = tid; b < nb; b += DF_THREADS) {
    const float mb = mrow[b], sb = srow[b];
    M += mb;
    if (mb > 1e-30f) A += (double)(mb * __logf(mb));  // below 1e-30 the term is < 1e-28
    B += (double)(mb * sb);
    Z += (double)__expf(sb - smax);
  }
  M = df_block_sum(M, red);
  A = df_block_sum(A, red);
  B = df_block_sum(B, red);
  Z = df_block_sum(Z, red);
  if (tid == 0)
    kl[r] = (nb > 0 && M > 0.0) ? (float)(A / M - log(M) - B / M + (double)smax + log(Z)) : 0.f;
  if (teacher && nb > 0) {
    const float inv = M > 0.0 ? (float)(1.0 / M) : 0.f;
    float* trow = teacher + (long long)r * ldt;
    for (int b = tid; b < nb; b += DF_THREADS) trow[b] = mrow[b] * inv;
  }
}

long long mass_ld(const Geometry& g) { return ((long long)g.max_pos / 4 + 1 + 3) / 4 * 4; }

}  // namespace

bool distill_tc_shape(const Geometry& g) { return g.D == 128 && g.G == DK_G; }

size_t distill_tc_workspace_bytes(const Geometry& g) {
  return (size_t)2 * g.num_q * (size_t)mass_ld(g) * 4;  // block masses + indexer scores
}

cudaError_t launch_distill_tc(const Geometry& g, const void* q, const void* k_pool, const void* idx_q,
                              const void* idx_w, const void* kcomp, float* kl, float* lse, float* teacher,
                              int64_t ld, void* ws, cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  auto enc = tmap_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const long long ldm = mass_ld(g);
  float* mass = static_cast<float*>(ws);
  float* scores = mass + (long long)g.num_q * ldm;
  DkArgs a;
  a.q_seq = g.q_seq;
  a.q_pos = g.q_pos;
  a.page_table = g.page_table;
  a.num_q = g.num_q;
  a.batch = g.batch;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.max_pos = g.max_pos;
  a.Hq = g.Hq;
  a.scale_log2 = g.scale_log2;
  a.lse = lse;
  a.mass = mass;
  a.ldm = ldm;
  a.err = g.err;
  CUtensorMap tmQ, tmK;
  {
    cuuint64_t dims[3] = {128, (cuuint64_t)g.Hq, (cuuint64_t)g.num_q};
    cuuint64_t strides[2] = {256, (cuuint64_t)g.Hq * 256};
    cuuint32_t box[3] = {64, DK_G, DK_TQ};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {128, (cuuint64_t)g.Hkv, (cuuint64_t)g.num_pages * 64};
    cuuint64_t strides[2] = {256, (cuuint64_t)g.Hkv * 256};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(k_pool), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaMemsetAsync(mass, 0, (size_t)g.num_q * ldm * 4, s);
  if (e != cudaSuccess) return e;
  if ((e = set_smem_once(distill_tc_kernel, DK_SMEM)) != cudaSuccess) return e;
  const int nt = DK_NQ * DK_TQ;
  distill_tc_kernel<<<dim3((g.num_q + nt - 1) / nt, g.Hkv), DK_THREADS, DK_SMEM, s>>>(a, tmQ, tmK);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_scores_only(g, idx_q, idx_w, kcomp, scores, ldm, s)) != cudaSuccess) return e;
  distill_finish_kernel<<<g.num_q, DF_THREADS, 0, s>>>(a, scores, ldm, kl, teacher, ld);
  return cudaGetLastError();
}

}  // namespace qsa
