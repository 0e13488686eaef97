// Steps (b)+(c): indexer block scoring and exact top-k selection.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token window
// with a selective view": four indexer query heads score the compressed micro-blocks of the one
// shared key head, the best 512 micro-blocks are kept (a 2,048-token budget, the same at every
// context length) together with the unfinished block at the sequence tail.  Library readings:
// s_b(t) = sum_h w_h(t) * max(0, q_h(t) . k_b) with bf16 operands and fp32 accumulation;
// candidates are b < t/4; ties go to the lower block index; the tail block t/4 is always kept.
//
// Two algorithms, same result:
//  * streaming (many query rows, e.g. a 16,384-token prefill chunk at 1M context, where the full
//    score matrix would be 17 GB): a CTA owns 64 query rows of one sequence and streams every
//    compressed-key tile of that sequence through shared memory once; tensor-core MMAs produce
//    the four head scores of 64 rows x 64 blocks, the epilogue applies ReLU, the head weights and
//    the causal limit, and appends every key above the row's running threshold to a per-row
//    candidate buffer; a full buffer is cut back to the exact top-k by a warp radix select, which
//    also raises the threshold.
//  * materialised (few query rows, any Di): all SMs split the block range, write fp32 scores
//    (16 MiB at 4 sequences x 4 positions x 1M context, L2-resident), then a histogram of the top
//    11 bits of the ordered score finds the bucket holding the k-th score, a filter pass collects
//    the keys above/in that bucket, and one CTA per row finishes the exact selection.
//  * split lists (few query rows, Di = 128; score_dec.cu): every warp streams a chunk of pages
//    and keeps each row's 32 best keys of its chunk; one CTA per row merges the lists exactly.
// The tensor-core (score_tc.cu) and split-list kernels flag rows they cannot settle exactly; the
// streaming kernel recomputes just those rows.
#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "score_common.cuh"

#include <algorithm>

namespace qsa {
namespace {

// =============================================================================== streaming

constexpr int ST_ROWS = 64;
constexpr int ST_THREADS = 256;
constexpr int ST_NST = 2;

__host__ __device__ constexpr int stream_cap(int topk) {
  // candidate slots per row: room for one tile of inserts after a cut back to topk
  return ((4 * topk > topk + 128 ? 4 * topk : topk + 128) + 63) / 64 * 64;
}

template <int DI>
struct StreamSmem {
  static constexpr int Q = 4 * ST_ROWS * DI * 2;
  static constexpr int B = ST_NST * 64 * DI * 2;
  static constexpr int SORT = 8 * 512 * 8;
  static constexpr int BIG = Q + (B > SORT ? B : SORT);  // sort scratch reuses the B tiles only
  static constexpr int W = ST_ROWS * 4 * 4;
  static constexpr int ROWI = ST_ROWS * 4 * 4;  // lim, seq, cnt, pos
  static constexpr int THR = ST_ROWS * 8;
  static constexpr int HIST = 8 * 256 * 4;
  static constexpr int MISC = 64;
  static constexpr int TOTAL = BIG + W + ROWI + THR + HIST + MISC;
};

template <int DI>
__global__ void __launch_bounds__(ST_THREADS, 2)
    score_stream_kernel(ScoreArgs a, u64* __restrict__ cand, int cap, const int32_t* redo) {
  chain_wait();
  chain_release();
  using S = StreamSmem<DI>;
  constexpr int CH = DI / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  bf16* sQ = reinterpret_cast<bf16*>(smem);                        // [4][64][DI]
  const uint32_t sQa = smem_addr(sQ);
  const uint32_t sBa = sQa + S::Q;                                  // [NST][64][DI]
  float* sW = reinterpret_cast<float*>(smem + S::BIG);              // [64][4]
  int* sLim = reinterpret_cast<int*>(sW + ST_ROWS * 4);             // [64]
  int* sSeq = sLim + ST_ROWS;                                        // [64]
  int* sCnt = sSeq + ST_ROWS;                                        // [64]
  int* sPosv = sCnt + ST_ROWS;                                       // [64]
  u64* sThr = reinterpret_cast<u64*>(sPosv + ST_ROWS);              // [64]
  uint32_t* sHist = reinterpret_cast<uint32_t*>(sThr + ST_ROWS);    // [8][256]
  int* sMisc = reinterpret_cast<int*>(sHist + 8 * 256);             // need[2], seg, nb

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * ST_ROWS;

  // redo != nullptr: only rows with redo[row] != 0 are computed (rows another kernel could not
  // finish); every other row is left untouched.
  if (tid < ST_ROWS) {
    const int r = row0 + tid;
    int seq = -1, lim = -1;
    bool skip = false;
    if (r < a.num_q) {
      if (redo && redo[r] == 0) skip = true;
      else lim = row_limit(a, r, &seq);
    }
    sSeq[tid] = lim >= 0 ? seq : -1;
    sPosv[tid] = skip ? -2 : lim;
  }
  if (tid < 4) sMisc[tid] = 0;
  __syncthreads();
  {
    bool any = false;
    for (int r = 0; r < ST_ROWS; ++r) any |= sSeq[r] >= 0;
    if (!any && redo) return;  // nothing to redo in this tile (uniform over the CTA)
  }
  for (int r = warp * 8; r < warp * 8 + 8; ++r)
    if (row0 + r < a.num_q && sPosv[r] == -1)
      write_empty_selection(row0 + r, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
  for (int i = tid; i < ST_ROWS * kHi * CH; i += ST_THREADS) {
    const int row = i / (kHi * CH), h = (i / CH) % kHi, c = i % CH;
    const bool valid = row0 + row < a.num_q;
    const bf16* src = valid ? a.idx_q + ((long long)(row0 + row) * kHi + h) * DI + c * 8 : a.idx_q;
    cp_async16(sQa + h * (ST_ROWS * DI * 2) + swz<DI>(row, c), src, valid);
  }
  cp_async_commit();
  {
    const int row = tid >> 2, h = tid & 3;
    sW[tid] = (row0 + row < a.num_q) ? __bfloat162float(a.idx_w[(long long)(row0 + row) * kHi + h]) : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();

  const int rg = warp & 3;       // row group: rows rg*16 .. +16
  const int bh = warp >> 2;      // block half of each 64-block tile
  const int r0 = rg * 16 + (lane >> 2), r1 = r0 + 8;
  float w0[4], w1[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    w0[h] = sW[r0 * 4 + h];
    w1[h] = sW[r1 * 4 + h];
  }

  for (;;) {
    // ---- pick the next sequence segment of this row tile
    __syncthreads();
    if (tid == 0) {
      int seg = -1;
      for (int r = 0; r < ST_ROWS; ++r)
        if (sSeq[r] >= 0) { seg = sSeq[r]; break; }
      sMisc[2] = seg;
    }
    __syncthreads();
    const int seg = sMisc[2];
    if (seg < 0) break;
    if (tid < ST_ROWS) {
      const bool act = sSeq[tid] == seg;
      sLim[tid] = act ? sPosv[tid] : -1;  // -1: not in this segment
      sCnt[tid] = 0;
      sThr[tid] = 0ull;
      if (act) sSeq[tid] = -1;
    }
    __syncthreads();
    if (tid == 0) {
      int nb = 0;
      for (int r = 0; r < ST_ROWS; ++r) nb = max(nb, sLim[r]);
      sMisc[3] = nb;
    }
    __syncthreads();
    const int nb = sMisc[3];
    const int lim0 = sLim[r0], lim1 = sLim[r1];
    const int ntiles = (nb + 63) / 64;

    for (int s = 0; s < ST_NST - 1; ++s) {
      if (s < ntiles) load_kcomp_tile<DI, ST_THREADS>(a, seg, s, nb, sBa + s * (64 * DI * 2));
      cp_async_commit();
    }
    for (int tile = 0; tile < ntiles; ++tile) {
      cp_async_wait<ST_NST - 2>();
      __syncthreads();  // tile landed; previous tile fully consumed; its inserts are done
      {
        const int nt = tile + ST_NST - 1;
        if (nt < ntiles) load_kcomp_tile<DI, ST_THREADS>(a, seg, nt, nb, sBa + (nt % ST_NST) * (64 * DI * 2));
        cp_async_commit();
      }
      const int pslot = (tile + 1) & 1;  // flag raised by the previous tile's epilogue
      if (sMisc[pslot]) {
        for (int r = warp * 8; r < warp * 8 + 8; ++r) {
          const int c = sCnt[r];
          if (c > cap - 64) {
            const u64 kth = warp_select_compact(cand + (long long)(row0 + r) * cap, c, a.topk,
                                                sHist + warp * 256);
            if (lane == 0) {
              sCnt[r] = a.topk;
              sThr[r] = kth;
            }
          }
        }
        __syncthreads();
        if (tid == 0) sMisc[pslot] = 0;
      }
      const u64 thr0 = sThr[r0], thr1 = sThr[r1];
      const uint32_t sB = sBa + (tile % ST_NST) * (64 * DI * 2);

      float acc[4][4][4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[h][nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < DI / 16; ++ks) {
        uint32_t bfr[2][4];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const int brow = bh * 32 + p * 16 + (lane & 7) + ((lane >> 4) << 3);
          ldsm_x4(bfr[p], sB + swz<DI>(brow, ks * 2 + ((lane >> 3) & 1)));
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          uint32_t af[4];
          const int arow = rg * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          ldsm_x4(af, sQa + h * (ST_ROWS * DI * 2) + swz<DI>(arow, ks * 2 + (lane >> 4)));
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
            mma_bf16_16816(acc[h][nt], af, bfr[nt >> 1][(nt & 1) * 2], bfr[nt >> 1][(nt & 1) * 2 + 1]);
        }
      }
      // ---- epilogue: ReLU, head weights, causal limit, threshold, append
      const int bbase = tile * 64 + bh * 32 + 2 * (lane & 3);
      bool raise = false;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int b = bbase + nt * 8 + j;
          float s0 = w0[0] * fmaxf(acc[0][nt][j], 0.f);
          float s1 = w1[0] * fmaxf(acc[0][nt][2 + j], 0.f);
#pragma unroll
          for (int h = 1; h < 4; ++h) {
            s0 = fmaf(w0[h], fmaxf(acc[h][nt][j], 0.f), s0);
            s1 = fmaf(w1[h], fmaxf(acc[h][nt][2 + j], 0.f), s1);
          }
          if (b < lim0) {
            const u64 k = make_key(s0, (uint32_t)b);
            if (k > thr0) {
              const int p = atomicAdd(&sCnt[r0], 1);
              cand[(long long)(row0 + r0) * cap + p] = k;
              raise |= p >= cap - 64;
            }
          }
          if (b < lim1) {
            const u64 k = make_key(s1, (uint32_t)b);
            if (k > thr1) {
              const int p = atomicAdd(&sCnt[r1], 1);
              cand[(long long)(row0 + r1) * cap + p] = k;
              raise |= p >= cap - 64;
            }
          }
        }
      }
      if (raise) sMisc[tile & 1] = 1;
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- final exact selection, ascending sort, output (warp w: rows w*8 .. w*8+7)
    uint32_t* sblk = reinterpret_cast<uint32_t*>(smem + S::Q) + warp * 1024;
    float* ssc = reinterpret_cast<float*>(sblk + 512);
    for (int r = warp * 8; r < warp * 8 + 8; ++r) {
      const int lim = sLim[r];
      if (lim < 0) continue;
      u64* buf = cand + (long long)(row0 + r) * cap;
      int n = sCnt[r];
      if (n > a.topk) {
        warp_select_compact(buf, n, a.topk, sHist + warp * 256);
        n = a.topk;
      }
      __syncwarp();
      for (int i = lane; i < n; i += 32) {
        const u64 k = buf[i];
        sblk[i] = key_block(k);
        ssc[i] = key_score(k);
      }
      __syncwarp();
      warp_sort_blocks(sblk, ssc, n);
      write_selection(row0 + r, n, lim, sblk, ssc, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
      __syncwarp();
    }
  }
}

// =============================================================================== materialised

constexpr int MT_ROWS = 16;
constexpr int MT_THREADS = 128;
constexpr int MT_NST = 3;
constexpr int HIST_BINS = 2048;  // top 11 bits of the ordered fp32 score

template <int DI>
struct DenseSmem {
  static constexpr int Q = 4 * 16 * DI * 2;  // [row group][m = h*4 + rr][DI]
  static constexpr int B = MT_NST * 64 * DI * 2;
  static constexpr int TOTAL = Q + B + MT_ROWS * 4 * 4 + MT_ROWS * 4 * 3 + 32;
};

// scores[row * ld + b] for b < t/4.  Grid (ceil(num_q/16), R); CTA y covers blocks
// [y*chunk, (y+1)*chunk).  M = 16 rows of one MMA = 4 query rows x 4 heads (m = h*4 + rr).
template <int DI>
__global__ void __launch_bounds__(MT_THREADS)
    score_dense_kernel(ScoreArgs a, float* __restrict__ scores, long long ld, int chunk) {
  using S = DenseSmem<DI>;
  constexpr int CH = DI / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQa = smem_addr(smem);
  const uint32_t sBa = sQa + S::Q;
  float* sW = reinterpret_cast<float*>(smem + S::Q + S::B);  // [16][4]
  int* sLim = reinterpret_cast<int*>(sW + MT_ROWS * 4);       // [16]
  int* sSeq = sLim + MT_ROWS;
  int* sPosv = sSeq + MT_ROWS;
  int* sMisc = sPosv + MT_ROWS;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * MT_ROWS;
  const int blo = blockIdx.y * chunk;

  if (tid < MT_ROWS) {
    const int r = row0 + tid;
    int seq = -1, lim = -1;
    if (r < a.num_q) lim = row_limit(a, r, &seq);
    sSeq[tid] = lim >= 0 ? seq : -1;
    sPosv[tid] = lim;
  }
  for (int i = tid; i < MT_ROWS * kHi * CH; i += MT_THREADS) {
    const int row = i / (kHi * CH), h = (i / CH) % kHi, c = i % CH;
    const bool valid = row0 + row < a.num_q;
    const bf16* src = valid ? a.idx_q + ((long long)(row0 + row) * kHi + h) * DI + c * 8 : a.idx_q;
    const int grp = row >> 2, m = h * 4 + (row & 3);
    cp_async16(sQa + grp * (16 * DI * 2) + swz<DI>(m, c), src, valid);
  }
  cp_async_commit();
  if (tid < MT_ROWS * 4) {
    const int row = tid >> 2, h = tid & 3;
    sW[tid] = (row0 + row < a.num_q) ? __bfloat162float(a.idx_w[(long long)(row0 + row) * kHi + h]) : 0.f;
  }
  cp_async_wait<0>();
  __syncthreads();

  const int rr = (lane >> 2) & 3;  // query row within the group (C rows lane/4 and lane/4+8)
  const int hlo = lane >> 4;       // heads hlo and hlo+2 live in this lane

  for (;;) {
    __syncthreads();
    if (tid == 0) {
      int seg = -1;
      for (int r = 0; r < MT_ROWS; ++r)
        if (sSeq[r] >= 0) { seg = sSeq[r]; break; }
      sMisc[0] = seg;
      int nb = 0;
      if (seg >= 0)
        for (int r = 0; r < MT_ROWS; ++r)
          if (sSeq[r] == seg) nb = max(nb, sPosv[r]);
      sMisc[1] = nb;
    }
    __syncthreads();
    const int seg = sMisc[0];
    if (seg < 0) break;
    if (tid < MT_ROWS) {
      const bool act = sSeq[tid] == seg;
      sLim[tid] = act ? sPosv[tid] : -1;
      if (act) sSeq[tid] = -1;
    }
    __syncthreads();
    const int nb = sMisc[1];
    const int bhi = min(nb, blo + chunk);
    bool grp_act[4];
#pragma unroll
    for (int g = 0; g < 4; ++g)
      grp_act[g] = sLim[g * 4] >= 0 || sLim[g * 4 + 1] >= 0 || sLim[g * 4 + 2] >= 0 || sLim[g * 4 + 3] >= 0;
    int lim[4];
    float wa[4], wb[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      lim[g] = sLim[g * 4 + rr];
      wa[g] = sW[(g * 4 + rr) * 4 + hlo];
      wb[g] = sW[(g * 4 + rr) * 4 + hlo + 2];
    }
    const int t0 = blo / 64;
    const int ntiles = bhi > blo ? (bhi - 1) / 64 - t0 + 1 : 0;
    for (int s = 0; s < MT_NST - 1; ++s) {
      if (s < ntiles) load_kcomp_tile<DI, MT_THREADS>(a, seg, t0 + s, bhi, sBa + s * (64 * DI * 2));
      cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
      cp_async_wait<MT_NST - 2>();
      __syncthreads();
      {
        const int nt = it + MT_NST - 1;
        if (nt < ntiles) load_kcomp_tile<DI, MT_THREADS>(a, seg, t0 + nt, bhi, sBa + (nt % MT_NST) * (64 * DI * 2));
        cp_async_commit();
      }
      const uint32_t sB = sBa + (it % MT_NST) * (64 * DI * 2);
      const int tile = t0 + it;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (!grp_act[g]) continue;
        float acc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < DI / 16; ++ks) {
          uint32_t bfr[4], af[4];
          const int brow = warp * 16 + (lane & 7) + ((lane >> 4) << 3);
          ldsm_x4(bfr, sB + swz<DI>(brow, ks * 2 + ((lane >> 3) & 1)));
          const int m = (lane & 7) + (((lane >> 3) & 1) << 3);
          ldsm_x4(af, sQa + g * (16 * DI * 2) + swz<DI>(m, ks * 2 + (lane >> 4)));
          mma_bf16_16816(acc[0], af, bfr[0], bfr[1]);
          mma_bf16_16816(acc[1], af, bfr[2], bfr[3]);
        }
        const int row = row0 + g * 4 + rr;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          // this lane: heads hlo (c0,c1) and hlo+2 (c2,c3), blocks 2c and 2c+1
          const float p0 = fmaf(wb[g], fmaxf(acc[nt][2], 0.f), wa[g] * fmaxf(acc[nt][0], 0.f));
          const float p1 = fmaf(wb[g], fmaxf(acc[nt][3], 0.f), wa[g] * fmaxf(acc[nt][1], 0.f));
          const float send = hlo ? p0 : p1;
          const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
          const float s = __fadd_rn(hlo ? p1 + recv : p0 + recv, 0.0f);  // fold -0 onto +0
          const int b = tile * 64 + warp * 16 + nt * 8 + 2 * (lane & 3) + hlo;
          if (b < lim[g] && b < bhi) scores[(long long)row * ld + b] = s;
        }
      }
    }
    cp_async_wait<0>();
  }
}

// Workspace of the materialised path (per row): hist[2048] u32, counters (sure, bnd) u32,
// sure keys [512] u64, boundary keys [nbmax] u64.
struct MatWs {
  float* scores;
  uint32_t* hist;
  uint32_t* counters;
  u64* sure;
  u64* bnd;
  long long ld;
};

__global__ void mat_clear_kernel(MatWs w, int num_q) {
  const long long n = (long long)num_q * HIST_BINS;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    w.hist[i] = 0;
    if (i < 2LL * num_q) w.counters[i] = 0;
  }
}

__device__ __forceinline__ int row_lim_simple(const ScoreArgs& a, int r) {
  const int seq = a.q_seq[r], pos = a.q_pos[r];
  if (seq < 0 || seq >= a.batch || pos < 0 || pos / 64 >= a.max_pages || pos > a.max_pos) return -1;
  return pos / 4;
}

// Histogram of the top 11 bits of the ordered score; grid (num_q, S), 256 threads.
__global__ void __launch_bounds__(256) mat_hist_kernel(ScoreArgs a, MatWs w, int chunk) {
  __shared__ uint32_t h[HIST_BINS];
  const int row = blockIdx.x;
  const int lim = row_lim_simple(a, row);
  for (int i = threadIdx.x; i < HIST_BINS; i += 256) h[i] = 0;
  __syncthreads();
  const int lo = blockIdx.y * chunk, hi = min(lim, lo + chunk);
  const float* sc = w.scores + (long long)row * w.ld;
  for (int base = lo; base < hi; base += 256) {
    const int b = base + threadIdx.x;
    const float v = b < hi ? sc[b] : 0.f;
    hist_add(h, f32_to_ordered(v) >> 21, b < hi);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < HIST_BINS; i += 256)
    if (h[i]) atomicAdd(&w.hist[(long long)row * HIST_BINS + i], h[i]);
}

// Bucket holding the need-th largest score (need >= 1), from the row histogram; every thread of
// the block gets it.  Uses 256 threads x 8 bins, scanned from the top bin down.
__device__ int find_boundary_bin(const uint32_t* hist, uint32_t need, uint32_t* s_tot, int* s_out) {
  const int t = threadIdx.x;
  uint32_t c[8], tot = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = hist[HIST_BINS - 1 - 8 * t - j];
    tot += c[j];
  }
  s_tot[t] = tot;
  __syncthreads();
  if (t < 32) {  // exclusive prefix over the 256 thread totals, warp 0
    uint32_t v[8], sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = s_tot[t * 8 + j];
      sum += v[j];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
      if (t >= o) incl += x;
    }
    uint32_t run = incl - sum;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t x = v[j];
      s_tot[t * 8 + j] = run;  // exclusive prefix
      run += x;
    }
  }
  __syncthreads();
  const uint32_t excl = s_tot[t];
  if (excl < need && need <= excl + tot) {
    uint32_t acc = excl;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (acc + c[j] >= need) {
        *s_out = HIST_BINS - 1 - 8 * t - j;
        break;
      }
      acc += c[j];
    }
  }
  __syncthreads();
  return *s_out;
}

// Collect keys of bins above the boundary (sure) and in it (boundary); grid (num_q, S).
__global__ void __launch_bounds__(256) mat_filter_kernel(ScoreArgs a, MatWs w, int chunk) {
  __shared__ uint32_t s_tot[256];
  __shared__ int s_bin;
  const int row = blockIdx.x;
  const int lim = row_lim_simple(a, row);
  const int need = min(a.topk, lim);
  if (need <= 0) return;
  if (threadIdx.x == 0) s_bin = 0;
  const int bin = find_boundary_bin(w.hist + (long long)row * HIST_BINS, (uint32_t)need, s_tot, &s_bin);
  const int lo = blockIdx.y * chunk, hi = min(lim, lo + chunk);
  const float* sc = w.scores + (long long)row * w.ld;
  const int lane = threadIdx.x & 31;
  for (int base = lo; base < hi; base += 256) {
    const int b = base + threadIdx.x;
    u64 k = 0;
    int kb = -1;
    if (b < hi) {
      const float s = sc[b];
      k = make_key(s, (uint32_t)b);
      kb = (int)(f32_to_ordered(__fadd_rn(s, 0.0f)) >> 21);
    }
    const bool is_sure = kb > bin, is_bnd = kb == bin;
    const unsigned ms = __ballot_sync(0xffffffffu, is_sure);
    const unsigned mb = __ballot_sync(0xffffffffu, is_bnd);
    uint32_t bs = 0, bb = 0;
    if (lane == 0) {
      if (ms) bs = atomicAdd(&w.counters[2 * row], (uint32_t)__popc(ms));
      if (mb) bb = atomicAdd(&w.counters[2 * row + 1], (uint32_t)__popc(mb));
    }
    bs = __shfl_sync(0xffffffffu, bs, 0);
    bb = __shfl_sync(0xffffffffu, bb, 0);
    const unsigned lt = (1u << lane) - 1u;
    if (is_sure) w.sure[(long long)row * 512 + bs + __popc(ms & lt)] = k;
    if (is_bnd) w.bnd[(long long)row * w.ld + bb + __popc(mb & lt)] = k;
  }
}

// Exact finish: the (need - n_sure) largest boundary keys join the sure keys; sort ascending by
// block; write the selection.  One CTA (256 threads) per row.
__global__ void __launch_bounds__(256) mat_final_kernel(ScoreArgs a, MatWs w) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sblk[512];
  __shared__ float ssc[512];
  __shared__ int s_cnt;
  __shared__ int s_digit;
  __shared__ uint32_t s_above;
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int lim = row_lim_simple(a, row);
  if (lim < 0) {
    // invalid row: flagged by the score kernel; emit an empty selection
    if (tid < 32) write_empty_selection(row, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
    return;
  }
  const int need = min(a.topk, lim);
  const int n_sure = need > 0 ? (int)w.counters[2 * row] : 0;
  const int n_bnd = need > 0 ? (int)w.counters[2 * row + 1] : 0;
  const int rem = need - n_sure;
  const u64* bnd = w.bnd + (long long)row * w.ld;
  if (tid == 0) s_cnt = 0;
  __syncthreads();
  for (int i = tid; i < n_sure; i += 256) {
    const u64 k = w.sure[(long long)row * 512 + i];
    sblk[i] = key_block(k);
    ssc[i] = key_score(k);
  }
  if (rem > 0) {
    u64 kth = 0;  // keep boundary keys >= kth
    if (rem < n_bnd) {
      u64 prefix = 0, mask = 0;
      uint32_t remaining = (uint32_t)rem;
      for (int shift = 56; shift >= 0; shift -= 8) {
        hist[tid] = 0;
        __syncthreads();
        for (int base = 0; base < n_bnd; base += 256) {
          const int i = base + tid;
          const u64 k = i < n_bnd ? bnd[i] : 0ull;
          hist_add(hist, (uint32_t)(k >> shift) & 255u, i < n_bnd && (k & mask) == prefix);
        }
        __syncthreads();
        if (tid < 32) {
          uint32_t c[8], tot = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            c[j] = hist[255 - 8 * tid - j];
            tot += c[j];
          }
          uint32_t incl = tot;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (tid >= o) incl += v;
          }
          const uint32_t excl = incl - tot;
          if (excl < remaining && remaining <= incl) {
            uint32_t acc = excl;
            for (int j = 0; j < 8; ++j) {
              if (acc + c[j] >= remaining) {
                s_digit = 255 - 8 * tid - j;
                s_above = acc;
                break;
              }
              acc += c[j];
            }
          }
        }
        __syncthreads();
        remaining -= s_above;
        prefix |= (u64)s_digit << shift;
        mask |= 0xFFull << shift;
        __syncthreads();
      }
      kth = prefix;
    }
    for (int i = tid; i < n_bnd; i += 256) {
      const u64 k = bnd[i];
      if (k >= kth) {
        const int p = n_sure + atomicAdd(&s_cnt, 1);
        sblk[p] = key_block(k);
        ssc[p] = key_score(k);
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    warp_sort_blocks(sblk, ssc, need);
    write_selection(row, need, lim, sblk, ssc, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
  }
}

long long mat_ld(const Geometry& g) { return ((long long)(g.max_pos / 4 + 1) + 63) / 64 * 64; }

template <int DI>
cudaError_t run_dense_scores(const ScoreArgs& a, const Geometry& g, float* scores, long long ld,
                             cudaStream_t s) {
  const int tiles = (g.num_q + MT_ROWS - 1) / MT_ROWS;
  const long long nb = g.max_pos / 4 + 1;
  int R = (2 * num_sms() + tiles - 1) / tiles;
  long long chunk = (nb + R - 1) / R;
  chunk = (chunk + 63) / 64 * 64;
  if (chunk < 256) chunk = 256;
  R = (int)((nb + chunk - 1) / chunk);
  if (R < 1) R = 1;
  const int smem = DenseSmem<DI>::TOTAL;
  cudaError_t e = set_smem_once(score_dense_kernel<DI>, smem);
  if (e != cudaSuccess) return e;
  score_dense_kernel<DI><<<dim3(tiles, R), MT_THREADS, smem, s>>>(a, scores, ld, (int)chunk);
  return cudaGetLastError();
}

template <int DI>
cudaError_t run_stream(const ScoreArgs& a, const Geometry& g, void* ws, cudaStream_t s,
                       const int32_t* redo = nullptr) {
  const int smem = StreamSmem<DI>::TOTAL;
  cudaError_t e = set_smem_once(score_stream_kernel<DI>, smem);
  if (e != cudaSuccess) return e;
  const int tiles = (g.num_q + ST_ROWS - 1) / ST_ROWS;
  return launch_chained(score_stream_kernel<DI>, dim3(tiles), dim3(ST_THREADS), smem, s, a, static_cast<u64*>(ws),
                        stream_cap(g.topk), redo);
}

MatWs carve_mat(const Geometry& g, void* ws) {
  MatWs w;
  w.ld = mat_ld(g);
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](size_t bytes) {
    uint8_t* q = p;
    p += (bytes + 255) / 256 * 256;
    return q;
  };
  w.scores = reinterpret_cast<float*>(take((size_t)g.num_q * w.ld * 4));
  w.hist = reinterpret_cast<uint32_t*>(take((size_t)g.num_q * HIST_BINS * 4));
  w.counters = reinterpret_cast<uint32_t*>(take((size_t)g.num_q * 2 * 4));
  w.sure = reinterpret_cast<u64*>(take((size_t)g.num_q * 512 * 8));
  w.bnd = reinterpret_cast<u64*>(take((size_t)g.num_q * w.ld * 8));
  return w;
}

size_t mat_bytes(const Geometry& g) {
  const long long ld = mat_ld(g);
  auto r = [](size_t b) { return (b + 255) / 256 * 256; };
  return r((size_t)g.num_q * ld * 4) + r((size_t)g.num_q * HIST_BINS * 4) + r((size_t)g.num_q * 8) +
         r((size_t)g.num_q * 512 * 8) + r((size_t)g.num_q * ld * 8);
}

}  // namespace

// Path resolution is pure geometry, so workspace sizes are computable on a host with no driver.
int resolve_score_path(const Geometry& g, int requested) {
  switch (requested) {
    case 1: case 2: case 4: return requested;
    case 3: return score_dec_plan_ok(g) ? 3 : 2;
    case 5: return g.Di == 128 ? 5 : 1;
    default: break;
  }
  if (g.num_q <= 128 && score_dec_plan_ok(g)) return 3;
  if (g.num_q <= 256) return 2;
  return g.Di == 128 && !score_tc_stream_pays(g) ? 5 : 1;
}

// The fast Di = 128 kernels (tcgen05 prefill, split-list decode) load operands through tensor
// maps.  Without the driver's encoder they cannot run, and a silent switch to the mma.sync
// streaming kernel would be a large, invisible slowdown: the call reports it instead (path 4
// asks for the streaming kernel explicitly).
int tmap_encode_fn_available() { return tmap_encode_fn() != nullptr; }

bool score_path_runnable(const Geometry& g, int path) {
  const bool needs_tma = (path == 1 && g.Di == 128) || path == 3 || path == 5;
  return !needs_tma || tmap_encode_fn() != nullptr;
}

size_t score_workspace_bytes(const Geometry& g, int path) {
  if (path == 1 || path == 4 || path == 5) {
    size_t n = (size_t)g.num_q * stream_cap(g.topk) * 8;
    if (path == 1 && g.Di == 128) n = std::max(n, score_tc_workspace_bytes(g, true));
    if (path == 5) n = std::max(n, score_tc_workspace_bytes(g, false));
    return n;
  }
  if (path == 3) return score_dec_workspace_bytes(g);
  return mat_bytes(g);
}

bool score_redo_offset(const Geometry& g, int path, size_t* off) {
  if ((path == 1 && g.Di == 128) || path == 5) {
    *off = score_tc_redo_offset(g, path == 1);
    return true;
  }
  if (path == 3) {
    *off = score_dec_redo_offset(g);
    return true;
  }
  return false;
}

cudaError_t launch_score_topk(const Geometry& g, int path, const void* idx_q, const void* idx_w,
                              const void* kcomp, int32_t* sel, int32_t* n_sel, float* sel_scores,
                              void* ws, size_t ws_bytes, cudaStream_t s) {
  (void)ws_bytes;
  if (g.num_q == 0) return cudaSuccess;
  const ScoreArgs a = make_args(g, idx_q, idx_w, kcomp, sel, n_sel, sel_scores);
  if ((path == 1 && g.Di == 128) || path == 5) {
    // tensor-core kernels first (stream-K over every SM, or path 5: one CTA per 128-row tile);
    // the rows they flag are recomputed by the exact streaming kernel
    int32_t* redo = nullptr;
    cudaError_t e = launch_score_tc(a, g, ws, &redo, path == 1, s);
    if (e != cudaSuccess) return e;
    return run_stream<128>(a, g, ws, s, redo);
  }
  if (path == 1 || path == 4) {
    switch (g.Di) {
      case 32: return run_stream<32>(a, g, ws, s);
      case 64: return run_stream<64>(a, g, ws, s);
      default: return run_stream<128>(a, g, ws, s);
    }
  }
  if (path == 3) {  // the merge kernel runs the exact selection itself for rows it cannot settle
    int32_t* redo = nullptr;
    return launch_score_dec(a, g, ws, &redo, s);
  }
  MatWs w = carve_mat(g, ws);
  mat_clear_kernel<<<64, 256, 0, s>>>(w, g.num_q);
  cudaError_t e;
  switch (g.Di) {
    case 32: e = run_dense_scores<32>(a, g, w.scores, w.ld, s); break;
    case 64: e = run_dense_scores<64>(a, g, w.scores, w.ld, s); break;
    default: e = run_dense_scores<128>(a, g, w.scores, w.ld, s); break;
  }
  if (e != cudaSuccess) return e;
  const long long nb = g.max_pos / 4 + 1;
  int S = (4 * num_sms() + g.num_q - 1) / g.num_q;
  long long chunk = (nb + S - 1) / S;
  if (chunk < 2048) chunk = 2048;
  S = (int)((nb + chunk - 1) / chunk);
  if (S < 1) S = 1;
  mat_hist_kernel<<<dim3(g.num_q, S), 256, 0, s>>>(a, w, (int)chunk);
  mat_filter_kernel<<<dim3(g.num_q, S), 256, 0, s>>>(a, w, (int)chunk);
  mat_final_kernel<<<g.num_q, 256, 0, s>>>(a, w);
  return cudaGetLastError();
}

cudaError_t launch_scores_only(const Geometry& g, const void* idx_q, const void* idx_w,
                               const void* kcomp, float* scores, int64_t ld, cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  const ScoreArgs a = make_args(g, idx_q, idx_w, kcomp, nullptr, nullptr, nullptr);
  switch (g.Di) {
    case 32: return run_dense_scores<32>(a, g, scores, ld, s);
    case 64: return run_dense_scores<64>(a, g, scores, ld, s);
    default: return run_dense_scores<128>(a, g, scores, ld, s);
  }
}

}  // namespace qsa
