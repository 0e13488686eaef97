// Steps (b)+(c) on the 5th-generation tensor cores: indexer scoring with tcgen05.mma into TMEM,
// fused with ReLU, head weighting, the causal limit and candidate filtering for the exact top-k.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token window
// with a selective view": four indexer query heads score every compressed micro-block of the one
// shared key head and the best 512 are kept.  At a 1M-token context a 16,384-token prefill chunk is
// a [65,536 x 128] x [128 x 262,144] bf16 contraction (4.4 TFLOP) whose 17 GB score matrix must
// never be stored, so the selection is fused into the epilogue.
//
// CTA = 128 query rows (M = 128, one sequence segment at a time), warp-specialised:
//   warp 0      TMA producer: the 4 heads' query tiles (128 KB), then 128-block tiles of the
//               compressed keys (8 pages x 2 K-halves of 16 rows x 128 B, 128-byte swizzle) into a
//               3-stage ring (96 KB);
//   warp 1      owns the TMEM allocation (512 columns: pair X = heads 0,1 and pair Y = heads 2,3,
//               each 2 x 128 blocks) and one lane issues 2 x 8 tcgen05.mma (M=128, N=128, K=16)
//               into X, then 2 x 8 into Y, per tile; N=128 keeps the tensor pipe fed from shared
//               memory (each MMA re-reads its 4 KB query slice for 2x the work of N=64);
//   warps 2-9   epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (= its 32 query rows) and half of
//               the 128 columns; thread = (query row, column half).  The weighted ReLU sum of pair
//               X stays in registers while pair Y is computed, then X and Y are released in turn.
// Selection without in-loop compaction: the tile sequence is first every 32nd tile (a sample),
// then all tiles.  During the sample each thread keeps the TC_KEEP = 24 best sampled scores of
// its half-row in registers; the row threshold tau = min over its two halves of the 24th best, so
// about 1,700 of the row's scores are >= tau (on independent scores: mean 1,711-1,727, standard
// deviation 260-274 at 32K-262K candidates) and fewer than 512 is a more than 4-sigma event.  Each
// kept key costs an append and a share of the final select, so a lower rank is faster until the
// exact fallback starts to be needed.  Rows of at most 2 * TC_CAP candidates skip the threshold
// and keep every key (a sample of one or two tiles would keep too few).  The full pass appends
// every (score >= tau, block) key to a per-half-row buffer (in ascending block order); the final
// step checks that at least min(512, t/4) keys were kept -- which proves every true top-512 key
// was kept -- and selects exactly (radix select on 64-bit keys, lower block index wins ties) and
// merges the two lists by block.  Rows that fail the check (adversarial score orders) or overflow
// the buffer are recomputed by the exact streaming kernel, so the result never depends on the
// sample.
#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"
#include "select.cuh"
#include "tc_common.cuh"

namespace qsa {
namespace {

constexpr int TC_ROWS = 128;
constexpr int TC_BLK = 128;           // blocks per tile (MMA N)
constexpr int TC_PG = TC_BLK / 16;    // pages per tile
constexpr int TC_NST = 3;             // compressed-key stages
constexpr int TC_SAMPLE = 32;         // every 32nd tile is sampled
constexpr int TC_KEEP = 24;           // best sampled scores kept per half-row (threshold rank)
constexpr int TC_EPI = 8;             // epilogue warps
constexpr int TC_THREADS = (2 + TC_EPI) * 32;
constexpr int TC_A_BYTES = 4 * 2 * TC_ROWS * 128;  // 4 heads x 2 K-halves x 128 rows x 128 B
constexpr int TC_B_STAGE = 2 * TC_BLK * 128;       // 2 K-halves x 128 rows x 128 B
constexpr int TC_B_BYTES = TC_NST * TC_B_STAGE;
constexpr int TC_CAP = 2048;          // candidate slots per half-row
constexpr int TC_STREAM_CTAS = 148;   // CTAs of the stream-K launch (one per SM of a B200)

// The three launches of the stream-K form (mode 0 is the single-launch form):
//   mode 1  sample: per row tile, the sampled threshold of every row (tau), the number of full
//           tiles of the row tile (tiles), empty selections of invalid rows, cleared redo flags;
//   mode 2  stream: CTA c takes the full tiles [c W, (c+1) W) of the concatenation of every row
//           tile's tiles (W = ceil(total / TC_STREAM_CTAS)); the part of row tile r that CTA c
//           covers is an item, and items are numbered r + c (unique: the CTAs' ranges follow
//           one another, so a later row tile never meets an earlier CTA); each item keeps, per
//           row and column half, its keys at or above tau in block order (runs, runcnt);
//   select  (tc_select_kernel) per row: the item runs of its row tile in CTA order, so that each
//           column half's list is ascending by block, then the exact select.
struct TcPlan {
  int mode;
  float* tau;             // [num_q]
  int32_t* tiles;         // [R]
  int32_t* prefix;        // [R + 1]: exclusive prefix of tiles, the total last
  int32_t* runcnt;        // [(R + TC_STREAM_CTAS) * 128 * 2]
  u64* runs;              // [(R + TC_STREAM_CTAS) * 128 * 2 * TC_CAP]
};

struct TcMisc {
  // tfull/tempty[0]: TMEM pair X (heads 0, 1); [1]: pair Y (heads 2, 3)
  uint64_t full[TC_NST], empty[TC_NST], tfull[2], tempty[2], aload, mma_done;
  uint64_t stage[TC_EPI];  // final select: bulk copies of one row's candidate keys, per warp
  uint32_t tmem_base;
  int abort_flag;
  int issued, consumed;  // B tiles issued by the producer / waited for by the MMA issuer
  int seg, nb;
  uint32_t done[4];      // rows already selected (bit per row)
  uint32_t inseg[4];     // rows of the current segment
  int lim[TC_ROWS];
  int cnt[2][TC_ROWS];
  float thr[2][TC_ROWS];
  int tiles_acc;  // mode 1: full tiles of the row tile's segments
};
// operands + bookkeeping; the dynamic shared-memory base must be 1024-byte aligned (checked)
constexpr int TC_SMEM = TC_A_BYTES + TC_B_BYTES + (int)((sizeof(TcMisc) + 127) / 128 * 128);
static_assert(TC_SMEM <= 232448, "shared memory budget");

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M=128, N=128.
constexpr uint32_t kIdesc = idesc_bf16(TC_ROWS, TC_BLK, false);

// Packed fp32 pairs (sm_100): one instruction rounds both lanes exactly as the scalar op would.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(TC_EPI * 32)); }

__device__ __forceinline__ bool bit_of(const uint32_t* b, int i) { return (b[i >> 5] >> (i & 31)) & 1u; }

// v[base + j] for a run-time j in 0..31, out of registers: a 5-level select tree (31 selects, 5
// deep) instead of a chain of 31 dependent selects.
__device__ __forceinline__ float pick32(const float (&v)[64], int base, int j) {
  float l1[16], l2[8], l3[4], l4[2];
#pragma unroll
  for (int k = 0; k < 16; ++k) l1[k] = (j & 1) ? v[base + 2 * k + 1] : v[base + 2 * k];
#pragma unroll
  for (int k = 0; k < 8; ++k) l2[k] = (j & 2) ? l1[2 * k + 1] : l1[2 * k];
#pragma unroll
  for (int k = 0; k < 4; ++k) l3[k] = (j & 4) ? l2[2 * k + 1] : l2[2 * k];
#pragma unroll
  for (int k = 0; k < 2; ++k) l4[k] = (j & 8) ? l3[2 * k + 1] : l3[2 * k];
  return (j & 16) ? l4[1] : l4[0];
}

// ------------------------------------------------------------------ final selection, one warp
// The row's candidate keys are staged in the warp's share of the (then idle) operand memory:
// sk[0..n0) from column half 0 and sk[n0..n0+n1) from column half 1, each list ascending by
// block.  Shared memory keeps every pass of the select at shared-memory latency.
constexpr int TC_SEL_REGION = (TC_A_BYTES + TC_B_BYTES) / TC_EPI;  // bytes per epilogue warp
constexpr int TC_SEL_HIST = 256;                                  // 8-bit digits
constexpr int TC_SEL_KEYS = (TC_SEL_REGION - TC_SEL_HIST * 4) / 8;
static_assert(TC_SEL_REGION % 16 == 0 && TC_SEL_REGION >= 2048 * 4, "selection region");

// The need-th largest of the n unique keys sk[0..n), 1 <= need <= n: MSB-first radix select with
// 8-bit digits starting at the highest bit where the keys differ; stops as soon as the digit's
// bucket is kept whole (its smallest key is then the answer).
__device__ __forceinline__ u64 tc_kth_largest(const u64* sk, int n, int need, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  u64 lo = ~0ull, hi = 0ull;
  for (int i = lane; i < n; i += 32) {
    const u64 k = sk[i];
    lo = k < lo ? k : lo;
    hi = k > hi ? k : hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const u64 x = __shfl_xor_sync(0xffffffffu, lo, o), y = __shfl_xor_sync(0xffffffffu, hi, o);
    lo = x < lo ? x : lo;
    hi = y > hi ? y : hi;
  }
  if (need == n) return lo;
  if (need == 1) return hi;
  int top = 63 - __clzll((long long)(lo ^ hi));  // lo != hi: n >= 2 unique keys
  u64 mask = top == 63 ? 0ull : ~((2ull << top) - 1ull);
  u64 prefix = hi & mask;
  uint32_t remaining = (uint32_t)need;
  for (;;) {
    const int width = top + 1 < 8 ? top + 1 : 8;
    const int shift = top + 1 - width;
    const uint32_t dmask = (1u << width) - 1u;
#pragma unroll
    for (int j = 0; j < TC_SEL_HIST / 32; ++j) hist[j * 32 + lane] = 0;
    __syncwarp();
    for (int b0 = 0; b0 < n; b0 += 128) {  // four loads in flight per lane, then the atomics
      u64 k[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = b0 + u * 32 + lane;
        k[u] = i < n ? sk[i] : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = b0 + u * 32 + lane;
        if (i < n && (k[u] & mask) == prefix) atomicAdd(&hist[(uint32_t)(k[u] >> shift) & dmask], 1u);
      }
    }
    __syncwarp();
    // lane l owns bins 255-8l down to 248-8l, counted from the top; the sum reads them in a
    // lane-staggered order, so the 32 lanes hit 32 different banks
    uint32_t tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) tot += hist[255 - 8 * lane - ((j + (lane >> 2)) & 7)];
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const bool mine = excl < remaining && remaining <= incl;
    int digit = 0;
    uint32_t above = 0, cnt_at = 0;
    if (mine) {
      uint32_t acc = excl;
      for (int j = 0; j < 8; ++j) {
        const uint32_t c = hist[255 - 8 * lane - j];
        if (acc + c >= remaining) {
          digit = 255 - 8 * lane - j;
          above = acc;
          cnt_at = c;
          break;
        }
        acc += c;
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    cnt_at = __shfl_sync(0xffffffffu, cnt_at, src);
    remaining -= above;
    prefix |= (u64)digit << shift;
    mask |= (u64)dmask << shift;
    __syncwarp();
    if (shift == 0) return prefix;
    if (cnt_at == remaining) {  // the whole bucket is kept: the answer is its smallest key
      u64 m = ~0ull;
      for (int i = lane; i < n; i += 32) {
        const u64 k = sk[i];
        if ((k & mask) == prefix && k < m) m = k;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const u64 x = __shfl_xor_sync(0xffffffffu, m, o);
        m = x < m ? x : m;
      }
      return m;
    }
    top = shift - 1;
  }
}

// Keep the keys >= kth of s[0..n), compacted in place in their order; returns how many.
__device__ __forceinline__ int tc_keep_inplace(u64* s, int n, u64 kth) {
  const int lane = threadIdx.x & 31;
  int w = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const u64 k = i < n ? s[i] : 0ull;
    const bool keep = i < n && k >= kth;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);  // every lane has read before any writes
    if (keep) s[w + __popc(bal & ((1u << lane) - 1u))] = k;
    w += __popc(bal);
    __syncwarp();
  }
  return w;
}

// The selection row from two disjoint lists of kept keys, each ascending by block (a larger low
// word is a smaller block): a merge path, each lane writing a contiguous run of output positions,
// then the tail block and the padding.
__device__ __forceinline__ void tc_write_merged(const u64* A, int na, const u64* B, int nb, int row,
                                                int tail, const ScoreArgs& a) {
  const int lane = threadIdx.x & 31;
  const int n = na + nb;
  int32_t* srow = a.sel + (long long)row * a.sel_stride;
  float* crow = a.sel_scores ? a.sel_scores + (long long)row * a.sel_stride : nullptr;
  auto before = [](u64 x, u64 y) { return (uint32_t)x > (uint32_t)y; };  // block(x) < block(y)
  const int per = (n + 31) >> 5;
  const int d0 = min(lane * per, n), d1 = min(d0 + per, n);
  int lo = max(0, d0 - nb), hi = min(d0, na);
  while (lo < hi) {  // how many of the first d0 outputs come from A
    const int mid = (lo + hi) >> 1;
    if (before(A[mid], B[d0 - mid - 1])) lo = mid + 1;
    else hi = mid;
  }
  int i = lo, j = d0 - lo;
  for (int d = d0; d < d1; ++d) {
    const bool takeA = j >= nb || (i < na && before(A[i], B[j]));
    const u64 k = takeA ? A[i++] : B[j++];
    srow[d] = (int32_t)key_block(k);
    if (crow) crow[d] = key_score(k);
  }
  for (int d = n + lane; d < a.sel_stride; d += 32) {
    srow[d] = d == n ? tail : -1;
    if (crow) crow[d] = d == n ? __int_as_float(0x7f800000) : __int_as_float(0x7fc00000);
  }
  if (lane == 0) a.n_sel[row] = n + 1;
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    score_tc_kernel(ScoreArgs a, const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, u64* __restrict__ cand,
                    int32_t* __restrict__ redo, TcPlan p) {
  chain_wait();  // before any global access and before the tensor-memory allocation
  chain_release();
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sA = smem;
  uint8_t* sB = smem + TC_A_BYTES;
  TcMisc* m = reinterpret_cast<TcMisc*>(sB + TC_B_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mode = p.mode;

  if (smem_addr(smem) & 1023) {  // operand tiles need 1024-byte alignment: leave the rows to the
    if (mode != 2 && tid < TC_ROWS && blockIdx.x * TC_ROWS + tid < a.num_q)  // exact streaming kernel
      redo[blockIdx.x * TC_ROWS + tid] = 1;
    if (tid == 0) flag_error(a.err, QSA_DEVERR_INTERNAL);
    return;
  }
  if (tid == 0) {
    for (int s = 0; s < TC_NST; ++s) {
      mbar_init(&m->full[s], 1);
      mbar_init(&m->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&m->tfull[b], 1);
      mbar_init(&m->tempty[b], TC_EPI);
    }
    mbar_init(&m->aload, 1);
    mbar_init(&m->mma_done, 1);
    for (int e = 0; e < TC_EPI; ++e) mbar_init(&m->stage[e], 1);
    m->abort_flag = 0;
    m->issued = 0;
    m->consumed = 0;
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

  // row tiles of this CTA: its own (modes 0, 1), or those its stream range meets (mode 2)
  int rt_begin = blockIdx.x, rt_end = blockIdx.x + 1;
  int g_lo = 0, g_hi = 0;  // mode 2: this CTA's range of full tiles
  if (mode == 2) {
    const int R = (a.num_q + TC_ROWS - 1) / TC_ROWS;
    const int total = p.prefix[R];
    const int W = (total + TC_STREAM_CTAS - 1) / TC_STREAM_CTAS;
    g_lo = min(blockIdx.x * W, total);
    g_hi = min(g_lo + W, total);
    rt_begin = rt_end = 0;
    if (g_lo < g_hi) {  // first row tile whose range ends after g_lo, last that starts before g_hi
      int lo = 0, hi = R;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (p.prefix[mid + 1] <= g_lo) lo = mid + 1;
        else hi = mid;
      }
      rt_begin = lo;
      rt_end = lo;
      while (rt_end < R && p.prefix[rt_end] < g_hi) ++rt_end;
    }
  }

  uint32_t stage_phase = 0;  // epilogue warps: phase of this warp's staging barrier
  bool stage_dead = false;   // a staging copy never landed: the warp's remaining rows go to redo
  int it_base = 0;  // tiles of earlier segments (all roles count the same tiles)
  int segi = 0;     // segments started (phase of the query-tile barrier)
  for (int rt = rt_begin; rt < rt_end; ++rt) {
  const int row0 = rt * TC_ROWS;
  // mode 2: the part of this row tile's tiles that the CTA covers, and its item slot
  const int r_lo = mode == 2 ? max(g_lo, p.prefix[rt]) - p.prefix[rt] : 0;
  const int r_hi = mode == 2 ? min(g_hi, p.prefix[rt + 1]) - p.prefix[rt] : 0;
  const int slot = rt + blockIdx.x;
  __syncthreads();  // the previous row tile's state is no longer read
  if (tid < TC_ROWS) {
    const int r = row0 + tid;
    int seq = -1, lim = -1;
    if (r < a.num_q) {
      lim = row_limit(a, r, &seq);
      if (mode != 2) redo[r] = 0;
    }
    m->lim[tid] = lim;
    const unsigned bal = __ballot_sync(0xffffffffu, lim < 0);  // invalid rows count as done
    if (lane == 0) m->done[tid >> 5] = bal;
    if (tid == 0) m->tiles_acc = 0;
  }
  if (mode == 2 && warp >= 2) {  // every row's run of this item starts empty
    const int rr = (warp & 3) * 32 + lane, hh = (warp - 2) >> 2;
    p.runcnt[((long long)slot * TC_ROWS + rr) * 2 + hh] = 0;
  }
  __syncthreads();
  if (mode != 2 && warp >= 2) {  // rows that failed validation get an empty selection
    for (int r = (warp - 2) * 16; r < (warp - 2) * 16 + 16; ++r)
      if (row0 + r < a.num_q && m->lim[r] < 0)
        write_empty_selection(row0 + r, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
  }
  int seg_off = 0;  // mode 2: this row tile's tiles before the current segment
  for (;;) {
    __syncthreads();
    if (warp == 0) {  // next segment: the sequence of the first row not yet done
      int seg = -1;
      for (int r = 0; r < TC_ROWS && seg < 0; ++r)
        if (!bit_of(m->done, r)) seg = a.q_seq[row0 + r];
      int nb = 0;
      for (int r = lane; r < TC_ROWS; r += 32) {
        const bool in = seg >= 0 && !bit_of(m->done, r) && a.q_seq[row0 + r] == seg;
        const unsigned bal = __ballot_sync(0xffffffffu, in);
        if (lane == 0) m->inseg[r >> 5] = bal;
        if (in) nb = max(nb, m->lim[r]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nb = max(nb, __shfl_xor_sync(0xffffffffu, nb, o));
      if (lane == 0) {
        m->seg = seg;
        m->nb = nb;
      }
    }
    __syncthreads();
    const int seg = m->seg;
    if (seg < 0 || m->abort_flag) break;
    const int ntile = (m->nb + TC_BLK - 1) / TC_BLK;
    // tiles of this segment in this launch: sample tiles, then full tiles [t_lo, t_hi)
    int nsamp = (ntile + TC_SAMPLE - 1) / TC_SAMPLE, t_lo = 0, t_hi = ntile;
    if (mode == 1) t_hi = 0;
    if (mode == 2) {
      nsamp = 0;
      t_lo = min(max(r_lo - seg_off, 0), ntile);
      t_hi = min(max(r_hi - seg_off, 0), ntile);
    }
    if (tid == 0) m->tiles_acc += ntile;
    seg_off += ntile;
    const int L = ntile > 0 ? nsamp + max(t_hi - t_lo, 0) : 0;
    if (mode == 2 && L == 0) {  // nothing of this segment here (every role sees the same)
      __syncthreads();
      if (tid < 4) m->done[tid] |= m->inseg[tid];
      continue;
    }

    if (warp == 0) {
      // ---------------------------------------------------------------- TMA producer
      // Page ids are fetched several tiles at a time, one per lane, so that no dependent
      // page-table load sits between two tile issues; lane 0 issues the copies.
      if (lane == 0) {  // query tiles, reloaded per segment (the final selection reuses sA)
        mbar_arrive_expect_tx(&m->aload, TC_A_BYTES);
        for (int h = 0; h < 4; ++h)
          for (int at = 0; at < 2; ++at)
            tma3d(smem_addr(sA + (h * 2 + at) * (TC_ROWS * 128)), &tmA, at * 64, h, row0, &m->aload);
      }
      const int32_t* pt = a.page_table + (long long)seg * a.max_pages;
      bool stop = false;
      for (int i0 = 0; i0 < L && !stop; i0 += 32 / TC_PG) {
        int mypage = 0;  // page slot lane%TC_PG of tile i0 + lane/TC_PG
        {
          const int i = i0 + lane / TC_PG;
          if (i < L) {
            const int tile = i < nsamp ? i * TC_SAMPLE : t_lo + i - nsamp;
            const int lp = tile * TC_PG + (lane % TC_PG);
            if (lp < a.max_pages) {  // pages past the table hold only masked blocks: page 0
              const int p = pt[lp];
              if (p >= 0 && p < a.num_pages) mypage = p;
              else flag_error(a.err, QSA_DEVERR_PAGE);
            }
          }
        }
        for (int j = 0; j < 32 / TC_PG; ++j) {
          const int i = i0 + j;
          int pgs[TC_PG];
#pragma unroll
          for (int pg = 0; pg < TC_PG; ++pg) pgs[pg] = __shfl_sync(0xffffffffu, mypage, j * TC_PG + pg);
          if (i >= L) break;
          if (lane == 0) {
            const int gi = it_base + i;
            const int s = gi % TC_NST;
            if (gi >= TC_NST && !mbar_wait(&m->empty[s], ((gi / TC_NST) & 1) ^ 1, a.err)) {
              m->abort_flag = 1;
              stop = true;
            } else {
              mbar_arrive_expect_tx(&m->full[s], TC_B_STAGE);
#pragma unroll
              for (int pg = 0; pg < TC_PG; ++pg)
#pragma unroll
                for (int at = 0; at < 2; ++at)
                  tma2d(smem_addr(sB + s * TC_B_STAGE + at * (TC_BLK * 128) + pg * 2048), &tmB, at * 64,
                        pgs[pg] * 16, &m->full[s]);
              m->issued = gi + 1;
            }
          }
          stop = __shfl_sync(0xffffffffu, stop, 0);
          if (stop) break;
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        bool ok = mbar_wait(&m->aload, segi & 1, a.err);
        for (int i = 0; ok && i < L; ++i) {
          const int gi = it_base + i;
          const int s = gi % TC_NST;
          if (!mbar_wait(&m->full[s], (gi / TC_NST) & 1, a.err)) { ok = false; break; }
          m->consumed = gi + 1;
          const uint32_t bst = smem_addr(sB + s * TC_B_STAGE);
#pragma unroll
          for (int pair = 0; pair < 2; ++pair) {
            // pair X (heads 0,1) -> columns 0..255, pair Y (heads 2,3) -> columns 256..511
            if (gi >= 1 && !mbar_wait(&m->tempty[pair], (gi - 1) & 1, a.err)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t ast = smem_addr(sA + (pair * 2 + hh) * 2 * (TC_ROWS * 128));
#pragma unroll
              for (int ks = 0; ks < 8; ++ks) {
                const uint64_t ad = sw128_desc(ast + (ks >> 2) * (TC_ROWS * 128) + (ks & 3) * 32);
                const uint64_t bd = sw128_desc(bst + (ks >> 2) * (TC_BLK * 128) + (ks & 3) * 32);
                umma_bf16(tbase + pair * 256 + hh * TC_BLK, ad, bd, kIdesc, ks > 0 ? 1u : 0u);
              }
            }
            umma_commit(&m->tfull[pair]);
          }
          if (!ok) break;
          umma_commit(&m->empty[s]);
        }
        if (!ok) m->abort_flag = 1;
      }
    } else {
      // ---------------------------------------------------------------- epilogue
      const int q = warp & 3;
      const int hf = (warp - 2) >> 2;
      const int row = q * 32 + lane;
      const int lim = bit_of(m->inseg, row) ? m->lim[row] : -1;
      float w[4];
#pragma unroll
      for (int h = 0; h < 4; ++h)
        w[h] = row0 + row < a.num_q ? __bfloat162float(a.idx_w[(long long)(row0 + row) * kHi + h]) : 0.f;
      float top[TC_KEEP];
#pragma unroll
      for (int k = 0; k < TC_KEEP; ++k) top[k] = -INFINITY;
      float mn = -INFINITY, tau = -INFINITY;
      int cnt = 0;
      u64* mybuf = mode == 2 ? p.runs + (((long long)slot * TC_ROWS + row) * 2 + hf) * TC_CAP
                             : cand + ((long long)(row0 + row) * 2 + hf) * TC_CAP;
      const uint32_t tl = tbase + ((uint32_t)(q * 32) << 16) + hf * 64;
      bool dead = false;
      // Scores of this thread's 64 blocks of tile gi: pair X folded into sc[] and released, then
      // pair Y added and released.
      auto load_scores = [&](int gi, float (&sc)[64]) -> bool {
        const uint32_t ph = gi & 1;
#pragma unroll
        for (int pair = 0; pair < 2; ++pair) {
          if (!dead && !mbar_wait(&m->tfull[pair], ph, a.err)) {
            m->abort_flag = 1;
            dead = true;
          }
          if (dead) return false;
          tc_fence_after();
          // two blocks per packed fp32x2 multiply / fma / add: wb*relu(vb) + wa*relu(va), the same
          // rounding steps as the scalar fmaf(wb, relu(vb), wa * relu(va))
          const uint64_t wa2 = pack_f32x2(w[pair * 2], w[pair * 2]);
          const uint64_t wb2 = pack_f32x2(w[pair * 2 + 1], w[pair * 2 + 1]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float va[16], vb[16];
            const uint32_t col = tl + pair * 256 + c * 16;
            tmem_ld16(col, va);
            tmem_ld16(col + TC_BLK, vb);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const uint64_t ra = pack_f32x2(fmaxf(va[j], 0.f), fmaxf(va[j + 1], 0.f));
              const uint64_t rb = pack_f32x2(fmaxf(vb[j], 0.f), fmaxf(vb[j + 1], 0.f));
              uint64_t x = fma_f32x2(wb2, rb, mul_f32x2(wa2, ra));
              if (pair == 1) x = add_f32x2(pack_f32x2(sc[c * 16 + j], sc[c * 16 + j + 1]), x);
              unpack_f32x2(x, sc[c * 16 + j], sc[c * 16 + j + 1]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&m->tempty[pair]);
        }
        return true;
      };
      // -- sample tiles: keep the TC_KEEP best scores of this half-row in registers.  The hot loop is
      // branch-free (bit masks of blocks above the current minimum); the rare insertions run from
      // one copy of the replacement code.
      for (int i = 0; i < nsamp && i < L; ++i) {
        float sc[64];
        if (!load_scores(it_base + i, sc)) continue;
        const int bbase = i * TC_SAMPLE * TC_BLK + hf * 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t hits = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            hits |= (uint32_t)(sc[half * 32 + j] > mn && bbase + half * 32 + j < lim) << j;
          while (hits) {
            const int j = __ffs(hits) - 1;
            hits &= hits - 1;
            const float x = pick32(sc, half * 32, j);
            if (x > mn) {  // replace one current minimum, then recompute the minimum
              bool done = false;
#pragma unroll
              for (int k = 0; k < TC_KEEP; ++k) {
                const bool hit = !done && top[k] == mn;
                top[k] = hit ? x : top[k];
                done |= hit;
              }
              mn = top[0];
#pragma unroll
              for (int k = 1; k < TC_KEEP; ++k) mn = fminf(mn, top[k]);
            }
          }
        }
      }
      // -- row threshold: every epilogue warp arrives here once per segment with tiles
      if (mode == 2) {
        tau = lim >= 0 ? p.tau[row0 + row] : -INFINITY;  // from the sample launch
      } else if (L > 0) {
        // a row of at most 2 * TC_CAP candidates keeps every key (each half-row holds at most
        // TC_CAP): a sample of one or two tiles would keep too few of them for the exact select
        m->thr[hf][row] = (lim > a.topk && lim > 2 * TC_CAP) ? mn : -INFINITY;
        epi_sync();
        tau = fminf(m->thr[0][row], m->thr[1][row]);
        if (mode == 1 && hf == 0 && lim >= 0) p.tau[row0 + row] = tau;
      }
      // -- all tiles: append every key with score >= tau (ascending block order per half-row)
      for (int i = nsamp; i < L; ++i) {
        float sc[64];
        if (!load_scores(it_base + i, sc)) continue;
        const int bbase = (t_lo + i - nsamp) * TC_BLK + hf * 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int nvalid = min(32, lim - bbase - half * 32);  // blocks below the causal limit
          uint32_t hits = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) hits |= (uint32_t)(sc[half * 32 + j] >= tau) << j;
          hits &= nvalid >= 32 ? 0xffffffffu : (nvalid <= 0 ? 0u : ((1u << nvalid) - 1u));
          while (hits) {  // ascending block order
            const int j = __ffs(hits) - 1;
            hits &= hits - 1;
            const float x = pick32(sc, half * 32, j);
            if (cnt < TC_CAP) mybuf[cnt] = make_key(x, (uint32_t)(bbase + half * 32 + j));
            ++cnt;
          }
        }
      }
      m->cnt[hf][row] = cnt;
      if (mode == 2 && lim >= 0) p.runcnt[((long long)slot * TC_ROWS + row) * 2 + hf] = cnt;
      // the final select reads the candidate buffers with bulk copies (async proxy)
      asm volatile("fence.proxy.async.global;\n" ::: "memory");
    }
    __syncthreads();  // the segment's tiles are all consumed; stage memory is free

    if (mode == 0 && warp >= 2 && !m->abort_flag) {
      // ---------------------------------------------------------------- exact final selection
      // Both half-row lists are ascending by block.  Find the need-th largest key of their union,
      // keep the keys >= it from each list in order, and merge the two by block.
      const int e = warp - 2;
      uint8_t* region = smem + e * TC_SEL_REGION;  // operand memory, idle until the next segment
      uint32_t* hist = reinterpret_cast<uint32_t*>(region);
      u64* sk = reinterpret_cast<u64*>(region + TC_SEL_HIST * 4);
      for (int rr = 0; rr < 16; ++rr) {
        const int row = e * 16 + rr;
        if (!bit_of(m->inseg, row)) continue;
        const int lim = m->lim[row];
        const int need = min(a.topk, lim);
        const int n0 = m->cnt[0][row], n1 = m->cnt[1][row];
        if (n0 > TC_CAP || n1 > TC_CAP || n0 + n1 < need) {
          if (lane == 0) redo[row0 + row] = 1;
          continue;
        }
        if (need == 0) {
          tc_write_merged(sk, 0, sk, 0, row0 + row, lim, a);
          __syncwarp();
          continue;
        }
        const u64* ka = cand + (long long)(row0 + row) * 2 * TC_CAP;
        const u64* kb = ka + TC_CAP;
        const int n0r = (n0 + 1) & ~1, n1r = (n1 + 1) & ~1;  // 16-byte multiples
        if (n0r + n1r <= TC_SEL_KEYS) {
          if (stage_dead) {
            if (lane == 0) redo[row0 + row] = 1;
            continue;
          }
          // stage sk = ka[0..n0) ++ [0 if n0 is odd] ++ kb[0..n1) with two bulk copies (both
          // lists start 16-byte aligned; a copy may read one stale key past a list's end, which
          // lies inside its buffer and is overwritten below)
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // after this warp's
          __syncwarp();                                                    // last use of sk
          if (lane == 0) {
            mbar_arrive_expect_tx(&m->stage[e], (uint32_t)(n0r + n1r) * 8u);
            if (n0r) bulk_g2s(smem_addr(sk), ka, (uint32_t)n0r * 8u, &m->stage[e]);
            if (n1r) bulk_g2s(smem_addr(sk + n0r), kb, (uint32_t)n1r * 8u, &m->stage[e]);
          }
          const bool landed = mbar_wait(&m->stage[e], stage_phase, a.err) ||
                              mbar_wait(&m->stage[e], stage_phase, a.err);  // bounded; 2nd: drain
          stage_phase ^= 1u;
          if (!landed) {  // (error flagged) the row goes to the exact kernel
            stage_dead = true;
            if (lane == 0) redo[row0 + row] = 1;
            continue;
          }
          if (lane == 0 && (n0 & 1)) sk[n0] = 0ull;  // below every key: never selected
          __syncwarp();
          const int n = n0r + n1;
          const u64 kth = tc_kth_largest(sk, n, need, hist);
          __syncwarp();
          const int na = tc_keep_inplace(sk, n0, kth);
          const int nb2 = tc_keep_inplace(sk + n0r, n1, kth);
          tc_write_merged(sk, na, sk + n0r, nb2, row0 + row, lim, a);
          __syncwarp();
          continue;
        }
        // more keys than the staging area holds: select from the (L2-resident) buffers in place
        uint32_t* h2 = reinterpret_cast<uint32_t*>(region);  // 2048 words, then the kept lists
        uint32_t* blk_a = h2;
        float* sc_a = reinterpret_cast<float*>(h2 + 512);
        uint32_t* blk_b = h2 + 1024;
        float* sc_b = reinterpret_cast<float*>(h2 + 1536);
        const u64 kth = warp_kth_largest2(ka, n0, kb, n0 + n1, need, h2);
        __syncwarp();
        const int na = warp_keep_sorted(ka, n0, kth, blk_a, sc_a);
        const int nb2 = warp_keep_sorted(kb, n1, kth, blk_b, sc_b);
        warp_write_merged(row0 + row, blk_a, sc_a, na, blk_b, sc_b, nb2, lim, a.sel, a.n_sel,
                          a.sel_scores, a.sel_stride);
        __syncwarp();
      }
      // the next segment's TMA copies overwrite this shared memory: order these generic accesses
      // before them
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    }
    __syncthreads();
    if (tid < 4) m->done[tid] |= m->inseg[tid];
    it_base += L;
    ++segi;
  }
  if (mode == 1 && tid == 0) p.tiles[rt] = m->tiles_acc;
  }  // row tiles

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (m->abort_flag && warp == 0 && lane == 0) {  // let copies still in flight land first
    if (segi > 0) mbar_wait(&m->aload, (segi - 1) & 1, a.err);
    for (int gi = m->consumed; gi < m->issued; ++gi)
      mbar_wait(&m->full[gi % TC_NST], (gi / TC_NST) & 1, a.err);
  }
  if (warp == 1) {
    if (lane == 0 && it_base > 0) {  // every issued MMA has completed before TMEM is released
      umma_commit(&m->mma_done);
      mbar_wait(&m->mma_done, 0, a.err);
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tbase));
  }
}

// Exclusive prefix of the row tiles' tile counts (one warp), the total last.
__global__ void tc_scan_kernel(const int32_t* __restrict__ tiles, int R, int32_t* __restrict__ prefix) {
  chain_wait();
  chain_release();
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < R; base += 32) {
    const int v = base + lane < R ? tiles[base + lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (base + lane < R) prefix[base + lane] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) prefix[R] = carry;
}

// The exact final select of the stream-K form, one warp per row: the runs its row tile's items
// left for the row, in CTA order (so that each column half's list is ascending by block, with a
// zero key after each odd-length run, below every real key), staged by bulk copies; then the
// need-th largest key, the keys at or above it kept in place, and a merge by block.
// Two warps (a pair) share one key area sized for the largest possible row: when both rows fit
// in it (the usual case: a row stages about 1,700 of the area's 4,394 slots) they run side by
// side, the odd warp's keys after the even warp's; otherwise the even warp runs first and hands
// the area over at the pair's barrier.  Sharing lets ten warps share an SM instead of six.
constexpr int TS_WARPS = 10;
constexpr int TS_KEYS = 2 * TC_CAP + 2 * (TC_STREAM_CTAS + 1);  // both halves, odd runs padded
constexpr int TS_RUNS = 2 * (TC_STREAM_CTAS + 1);                // runs of one row, at most
constexpr int TS_TABLE = (TS_RUNS * 8 + 15) / 16 * 16;           // (count, offset) per run
constexpr int TS_WARP_BYTES = TC_SEL_HIST * 4 + TS_TABLE;        // per warp: histogram, run table
constexpr int TS_SMEM = TS_WARPS * TS_WARP_BYTES + (TS_WARPS / 2) * TS_KEYS * 8;
static_assert(TS_WARPS % 2 == 0 && TS_WARPS / 2 <= 15, "warp pairs, one named barrier each");
static_assert(TS_WARP_BYTES % 16 == 0 && TS_SMEM <= 232448, "select shared memory");

__global__ void __launch_bounds__(TS_WARPS * 32) tc_select_kernel(ScoreArgs a, TcPlan p,
                                                                 int32_t* __restrict__ redo) {
  chain_wait();
  chain_release();
  extern __shared__ __align__(1024) uint8_t smem[];  // the one dynamic buffer of this file
  __shared__ uint64_t bar[TS_WARPS];
  __shared__ int pair_need[TS_WARPS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < TS_WARPS) mbar_init(&bar[threadIdx.x], 1);
  mbar_fence_init();
  __syncthreads();
  const int row = blockIdx.x * TS_WARPS + warp;
  uint8_t* region = smem + warp * TS_WARP_BYTES;
  uint32_t* hist = reinterpret_cast<uint32_t*>(region);
  int* table = reinterpret_cast<int*>(region + TC_SEL_HIST * 4);
  u64* pair_keys = reinterpret_cast<u64*>(smem + TS_WARPS * TS_WARP_BYTES) + (size_t)(warp >> 1) * TS_KEYS;

  // ---- this row's runs and staged size; rows with nothing to stage take no key slots
  bool work = false;
  int need = 0, lim = -1, nr = 0, c0 = 0, c1 = 0, rt = 0, rl = 0;
  int n[2] = {0, 0}, st[2] = {0, 0};
  if (row < a.num_q) {
    int seq = -1;
    lim = row_limit(a, row, &seq);  // < 0: the sample launch wrote its empty selection
    if (lim >= 0) need = min(a.topk, lim);
    if (lim >= 0 && need == 0) tc_write_merged(pair_keys, 0, pair_keys, 0, row, lim, a);  // no keys read
    if (lim >= 0 && need > 0) {
      const int R = (a.num_q + TC_ROWS - 1) / TC_ROWS;
      rt = row / TC_ROWS;
      rl = row % TC_ROWS;
      const int total = p.prefix[R];
      const int W = (total + TC_STREAM_CTAS - 1) / TC_STREAM_CTAS;
      const int S = p.prefix[rt], T = p.prefix[rt + 1] - S;
      if (T <= 0 || W <= 0) {  // no tile of this row was streamed: leave it to the exact kernel
        if (lane == 0) redo[row] = 1;
      } else {
        c0 = S / W;
        c1 = (S + T - 1) / W;
        nr = 2 * (c1 - c0 + 1);  // runs: half-major, then CTA order
        // every lane reads the counts of its runs at once; the staged slots follow by a warp scan
        for (int b0 = 0; b0 < nr; b0 += 32) {
          const int i = b0 + lane;
          const int h = i / (c1 - c0 + 1), c = c0 + i % (c1 - c0 + 1);
          const int k = i < nr ? p.runcnt[((long long)(rt + c) * TC_ROWS + rl) * 2 + h] : 0;
          const int kr = (min(k, TC_CAP) + 1) & ~1;
          int incl = kr;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
          }
          if (i < nr && i < TS_RUNS) {
            // staging offset of this run: the slots of every earlier run (earlier chunks included)
            const int off = st[0] + st[1] + incl - kr;
            table[2 * i] = k;  // (count, offset) of run i, for the copies and the pads below
            table[2 * i + 1] = off;
          }
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const bool mine = i < nr && h == h2;
            int kk = mine ? k : 0, ss = mine ? kr : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              kk += __shfl_xor_sync(0xffffffffu, kk, o);
              ss += __shfl_xor_sync(0xffffffffu, ss, o);
            }
            n[h2] += kk;
            st[h2] += ss;
          }
        }
        if (n[0] > TC_CAP || n[1] > TC_CAP || n[0] + n[1] < need || nr > TS_RUNS) {
          if (lane == 0) redo[row] = 1;
        } else {
          work = true;
        }
      }
    }
  }
  __syncwarp();

  // ---- the pair's key area: side by side when both rows fit, else the even warp first
  const int mine = work ? st[0] + st[1] : 0;  // even: 16-byte multiples of slots
  if (lane == 0) pair_need[warp] = mine;
  named_bar_sync(1 + (warp >> 1), 64);
  const int other = pair_need[warp ^ 1];
  const bool together = mine + other <= TS_KEYS;
  const bool even = (warp & 1) == 0;
  u64* sk = pair_keys + (together && !even ? other : 0);
  if (!together && !even) named_bar_sync(1 + (warp >> 1), 64);  // the even warp is done with it

  if (work) {
    // the area's earlier generic accesses (the partner's, in the sequential case) come before
    // the bulk copies' writes
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    if (lane == 0) mbar_arrive_expect_tx(&bar[warp], (uint32_t)(st[0] + st[1]) * 8u);
    __syncwarp();
    for (int i = lane; i < nr; i += 32) {  // one lane per run issues its copy
      const int h = i / (c1 - c0 + 1), c = c0 + i % (c1 - c0 + 1);
      const int k = table[2 * i], off = table[2 * i + 1];
      const int kr = (k + 1) & ~1;
      const long long base = ((long long)(rt + c) * TC_ROWS + rl) * 2 + h;
      if (kr) bulk_g2s(smem_addr(sk + off), p.runs + base * TC_CAP, (uint32_t)kr * 8u, &bar[warp]);
    }
    if (!mbar_wait(&bar[warp], 0, a.err)) {  // (error flagged) wait once more for the copies to land
      mbar_wait(&bar[warp], 0, a.err);
      if (lane == 0) redo[row] = 1;
    } else {
      for (int i = lane; i < nr; i += 32) {  // the slot after an odd run holds a stale key: below
        const int k = table[2 * i];          // every real key now
        if (k & 1) sk[table[2 * i + 1] + k] = 0ull;
      }
      __syncwarp();
      const u64 kth = tc_kth_largest(sk, st[0] + st[1], need, hist);
      __syncwarp();
      const int na = tc_keep_inplace(sk, st[0], kth);
      const int nb = tc_keep_inplace(sk + st[0], st[1], kth);
      tc_write_merged(sk, na, sk + st[0], nb, row, lim, a);
    }
  }
  __syncwarp();
  if (!together && even) named_bar_sync(1 + (warp >> 1), 64);  // hand the area to the odd warp
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tmap_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

namespace {
// Workspace of the stream-K form: runs | runcnt | tau | tiles | prefix | redo flags.
struct TcStreamWs {
  size_t runs, runcnt, tau, tiles, prefix, redo, total;
};
TcStreamWs stream_ws_layout(const Geometry& g) {
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t R = ((size_t)g.num_q + TC_ROWS - 1) / TC_ROWS;
  const size_t items = R + TC_STREAM_CTAS;
  TcStreamWs w;
  w.runs = 0;
  w.runcnt = w.runs + r256(items * TC_ROWS * 2 * TC_CAP * 8);
  w.tau = w.runcnt + r256(items * TC_ROWS * 2 * 4);
  w.tiles = w.tau + r256((size_t)g.num_q * 4);
  w.prefix = w.tiles + r256(R * 4);
  w.redo = w.prefix + r256((R + 1) * 4);
  w.total = w.redo + r256((size_t)g.num_q * 4);
  return w;
}
}  // namespace

// The stream-K form pays when the work it spreads over every SM saves more than its own costs
// (the sample and select launches, about 100 tiles' worth of one CTA): R row tiles of at most T
// key tiles take ceil(R / CTAs) * T tile times in the single-launch form, R * T / CTAs + 100 here.
// Pure geometry: T from the largest position.
bool score_tc_stream_pays(const Geometry& g) {
  const long long R = ((long long)g.num_q + TC_ROWS - 1) / TC_ROWS;
  const long long T = ((long long)g.max_pos / 4 + TC_BLK - 1) / TC_BLK + 1;
  const long long waves = (R + TC_STREAM_CTAS - 1) / TC_STREAM_CTAS;
  return R * T / TC_STREAM_CTAS + 100 < waves * T;
}

size_t score_tc_redo_offset(const Geometry& g, bool stream) {
  return stream ? stream_ws_layout(g).redo : (size_t)g.num_q * 2 * TC_CAP * 8;
}

size_t score_tc_workspace_bytes(const Geometry& g, bool stream) {
  if (stream) return stream_ws_layout(g).total;
  return score_tc_redo_offset(g, false) + ((size_t)g.num_q * 4 + 255) / 256 * 256;
}

// Launch the tensor-core kernel(s): the single-launch form (one CTA per 128-row tile) or the
// stream-K form (sample, scan, stream over every SM, select).  Rows they could not settle are
// flagged in `redo` (a workspace slice) for the exact streaming kernel, which the caller
// launches next.
cudaError_t launch_score_tc(const ScoreArgs& a, const Geometry& g, void* ws, int32_t** redo_out,
                            bool stream, cudaStream_t s) {
  auto enc = tmap_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  u64* cand = static_cast<u64*>(ws);
  int32_t* redo = reinterpret_cast<int32_t*>(wb + score_tc_redo_offset(g, stream));
  *redo_out = redo;
  CUtensorMap tmA, tmB;
  {
    cuuint64_t dims[3] = {128, 4, (cuuint64_t)g.num_q};
    cuuint64_t strides[2] = {256, 1024};
    cuuint32_t box[3] = {64, 1, TC_ROWS};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<bf16*>(a.idx_q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {128, (cuuint64_t)g.num_pages * 16};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(a.kcomp), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = set_smem_once(score_tc_kernel, TC_SMEM);
  if (e != cudaSuccess) return e;
  const int R = (g.num_q + TC_ROWS - 1) / TC_ROWS;
  TcPlan p{};
  if (!stream) {
    p.mode = 0;
    return launch_chained(score_tc_kernel, dim3(R), dim3(TC_THREADS), TC_SMEM, s, a, tmA, tmB, cand, redo, p);
  }
  const TcStreamWs w = stream_ws_layout(g);
  p.runs = reinterpret_cast<u64*>(wb + w.runs);
  p.runcnt = reinterpret_cast<int32_t*>(wb + w.runcnt);
  p.tau = reinterpret_cast<float*>(wb + w.tau);
  p.tiles = reinterpret_cast<int32_t*>(wb + w.tiles);
  p.prefix = reinterpret_cast<int32_t*>(wb + w.prefix);
  p.mode = 1;
  if ((e = launch_chained(score_tc_kernel, dim3(R), dim3(TC_THREADS), TC_SMEM, s, a, tmA, tmB, cand, redo, p)) !=
      cudaSuccess)
    return e;
  if ((e = launch_chained(tc_scan_kernel, dim3(1), dim3(32), 0, s, (const int32_t*)p.tiles, R, p.prefix)) !=
      cudaSuccess)
    return e;
  p.mode = 2;
  if ((e = launch_chained(score_tc_kernel, dim3(TC_STREAM_CTAS), dim3(TC_THREADS), TC_SMEM, s, a, tmA, tmB, cand,
                          redo, p)) != cudaSuccess)
    return e;
  if ((e = set_smem_once(tc_select_kernel, TS_SMEM)) != cudaSuccess) return e;
  return launch_chained(tc_select_kernel, dim3((g.num_q + TS_WARPS - 1) / TS_WARPS), dim3(TS_WARPS * 32), TS_SMEM, s,
                        a, p, redo);
}

}  // namespace qsa
