// Steps (b)+(c) for decode-sized batches (a few query rows per sequence, very long contexts):
// indexer scoring of every compressed micro-block with a split exact top-k.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token window
// with a selective view": four indexer query heads score every compressed micro-block of the one
// shared key head and the best 512 are kept, with the tail block.  At decode this is an HBM
// stream: each sequence's compressed keys (64 MiB at a 1M-token context, Di = 128) are read once
// for all of its query rows, and the arithmetic (16 query-head rows per block) is small.
//
// Kernel 1 (dec_score_kernel): query rows are taken four at a time (a "tile"; M = 16 MMA rows =
// 4 rows x 4 heads).  The pages of the tile's sequence are split into W contiguous chunks, one per
// warp, and warps are independent (no CTA barrier): each streams its pages (4 KB = 16 blocks x
// 128 dims, two 128-byte-swizzled TMA boxes) through a private 2-stage ring (16 warps per SM keep
// 128 KB in flight), scores them with
// mma.sync (the tile's query fragments stay in registers), applies ReLU, the head weights and the
// causal limit, and keeps for every row the exact 16 largest (score, block) keys of its chunk, as
// a list sorted across a half-warp (two rows per warp register): keys above the list's 16th key
// are appended to a 64-slot buffer, and a nearly full buffer is folded into the list by bitonic
// sort + merge networks over shuffles (15 exchange steps per 16 keys of each of two rows), which
// raises the threshold.
//
// Kernel 2 (dec_merge_kernel): one CTA per query row takes the union U of the row's W lists and
// selects its need = min(topk, t/4) largest keys exactly (CTA radix select).  That is the row's
// exact top-k whenever no list dropped a key that beats the need-th key of U: a list that dropped
// keys holds its chunk's 32 largest, so its dropped keys are all below its smallest kept key, and
// the check is smallest-kept <= tau for every such list.  With random scores a chunk would need
// more than 16 of the row's top 512 to fail (expected ~1); rows that fail are flagged for the exact
// streaming kernel, which the caller launches next, so the result never depends on the split.
#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"
#include "select.cuh"

namespace qsa {
namespace {

constexpr int DS_WARPS = 8;         // warps per CTA (independent while streaming)
constexpr int DS_THREADS = DS_WARPS * 32;
constexpr int DS_CTAS = 2;          // resident CTAs per SM (16 warps)
constexpr int DS_NST = 2;           // page stages per warp
constexpr int DS_KW = 16;           // keys kept per (warp chunk, row)
constexpr int DS_KC = 32;           // keys kept per (CTA chunk, row) when CTAs merge their warps
constexpr int DS_CAP = 64;          // candidate slots per (warp, row)
constexpr int DS_MAXPG = 256;       // pages per warp chunk
constexpr int DS_MINW = 128;        // warp chunks per tile when the context allows
constexpr int DS_MAXW = 1024;       // warp chunks per tile
constexpr int DS_CTA_MERGE_W = 512; // from this many warp chunks on, CTAs merge their warps' lists
constexpr int DS_PAGE = 16 * 128 * 2;  // one page of compressed keys, Di = 128
constexpr int DM_THREADS = 512;
constexpr int DM_MAXU = 8192;       // keys in one row's union
static_assert(DM_THREADS == 512 && 2 * DM_THREADS >= DS_MAXW,
              "16 warps; the list-offset scan takes two lists per thread");
static_assert(DS_MAXW / DS_WARPS * DS_KC <= DM_MAXU && (DS_CTA_MERGE_W - 1) * DS_KW <= DM_MAXU,
              "union bound");

struct DecSmem {
  static constexpr int STAGES = DS_WARPS * DS_NST * DS_PAGE;  // first, 1024-byte aligned
  static constexpr int BUF = DS_WARPS * 4 * DS_CAP * 8;
  static constexpr int MLIST = DS_WARPS * 4 * DS_KW * 8;      // warp lists for the CTA merge
  static constexpr int MBOUND = DS_WARPS * 4 * 8;
  static constexpr int PID = DS_WARPS * DS_MAXPG * 4;
  static constexpr int BAR = DS_WARPS * DS_NST * 8;
  static constexpr int TOTAL = STAGES + BUF + MLIST + MBOUND + PID + BAR + 1024;  // + alignment
};
static_assert(DS_CTAS * (DecSmem::TOTAL + 1024) <= 233472, "resident CTAs per SM");

struct DecPlan {
  int T;      // 4-row tiles
  int W;      // warp chunks per tile (a multiple of DS_WARPS: a CTA's warps share one tile)
  int chunk;  // pages per warp chunk
  int nl;     // lists per row handed to the merge: W, or W / DS_WARPS with the CTA merge
  int lk;     // keys per list: DS_KW, or DS_KC with the CTA merge
};

__host__ __device__ inline int pad2(int n) { return (n + 1) & ~1; }

// Chunking of the candidate pages: one warp per chunk, DS_CTAS CTAs per SM in total, at least
// DS_MINW chunks per tile (a row's union then holds >= 2,048 keys whenever any list dropped
// keys), chunks of at most DS_MAXPG pages.
bool dec_plan(const Geometry& g, DecPlan* p) {
  p->T = (g.num_q + 3) / 4;
  const long long pages = ((long long)g.max_pos / 4 + 15) / 16;  // candidates are b < t/4
  const long long P = pages > 0 ? pages : 1;
  long long W = ((long long)DS_CTAS * num_sms() * DS_WARPS + p->T - 1) / p->T;
  W = W < DS_MINW ? DS_MINW : (W > DS_MAXW ? DS_MAXW : W);
  if (W > P) W = P;
  long long chunk = (P + W - 1) / W;
  if (chunk > DS_MAXPG) chunk = DS_MAXPG;
  W = (P + chunk - 1) / chunk;
  W = (W + DS_WARPS - 1) / DS_WARPS * DS_WARPS;  // trailing chunks may be empty
  if (W > DS_MAXW) return false;
  p->W = (int)W;
  p->chunk = (int)chunk;
  const bool merge = W >= DS_CTA_MERGE_W;
  p->nl = merge ? p->W / DS_WARPS : p->W;
  p->lk = merge ? DS_KC : DS_KW;
  return true;
}

// Per query row, its nl lists are contiguous so that the merge fetches the row's union with one
// bulk copy: lists[row][l][lk] (descending, zero-padded) and bounds[row][pad2(nl)], where a
// list's bound is 0 if it kept every key of its chunk and otherwise a key above every dropped one.
struct DecWs {
  u64* lists;    // [T*4][nl][lk]
  u64* bounds;   // [T*4][pad2(nl)]
  int32_t* redo; // [num_q]
};

size_t r256(size_t b) { return (b + 255) / 256 * 256; }

// The exact streaming kernel's candidate buffers come first (it reuses the workspace base).
size_t stream_region(const Geometry& g) {
  const int topk = g.topk;
  const int cap = ((4 * topk > topk + 128 ? 4 * topk : topk + 128) + 63) / 64 * 64;
  return r256((size_t)g.num_q * cap * 8);
}

DecWs carve_dec(const Geometry& g, const DecPlan& p, void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws) + stream_region(g);
  DecWs w;
  w.lists = reinterpret_cast<u64*>(b);
  b += r256((size_t)p.T * 4 * p.nl * p.lk * 8);
  w.bounds = reinterpret_cast<u64*>(b);
  b += r256((size_t)p.T * 4 * pad2(p.nl) * 8);
  w.redo = reinterpret_cast<int32_t*>(b);
  return w;
}

// Bitonic exchange of one 64-bit key per lane with lane ^ j, keeping the max or the min.
__device__ __forceinline__ u64 cmpx(u64 v, int j, bool take_max) {
  const u64 o = __shfl_xor_sync(0xffffffffu, v, j);
  return take_max ? (o > v ? o : v) : (o < v ? o : v);
}

// Half-warp networks: lanes 0-15 and 16-31 each hold one row's list (rank = lane & 15,
// descending).  Sort the 16 keys of each half descending.
__device__ __forceinline__ u64 half_sort_desc(u64 v) {
  const int li = threadIdx.x & 15;
#pragma unroll
  for (int k = 2; k <= 16; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) v = cmpx(v, j, ((li & j) == 0) == ((li & k) == 0));
  return v;
}

// Fold up to 16 new keys per half into the half's list `top` (descending): the new keys are
// sorted, reversed against the list and maxed elementwise -- the best 16 of the two, as a bitonic
// sequence -- then bitonic-merged back into descending order.
__device__ __forceinline__ u64 half_merge16(u64 top, u64 v) {
  const int li = threadIdx.x & 15;
  v = half_sort_desc(v);
  const u64 rv = __shfl_xor_sync(0xffffffffu, v, 15);
  v = top > rv ? top : rv;
#pragma unroll
  for (int j = 8; j > 0; j >>= 1) v = cmpx(v, j, (li & j) == 0);
  return v;
}

// Whole-warp list of 32 (descending by lane): fold in two descending 16-lists held by the two
// halves.  Reversing the upper half makes the 32 keys bitonic; five merge steps sort them; then
// reversed-max against `top` and five more steps keep the best 32 of both.
__device__ __forceinline__ u64 warp_fold_two16(u64 top, u64 v) {
  const int lane = threadIdx.x & 31;
  const u64 r = __shfl_sync(0xffffffffu, v, 47 - lane);  // upper half reversed (lanes 16..31)
  if (lane >= 16) v = r;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) v = cmpx(v, j, (lane & j) == 0);
  const u64 rv = __shfl_sync(0xffffffffu, v, 31 - lane);
  v = top > rv ? top : rv;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) v = cmpx(v, j, (lane & j) == 0);
  return v;
}

__global__ void __launch_bounds__(DS_THREADS, DS_CTAS)
    dec_score_kernel(ScoreArgs a, const __grid_constant__ CUtensorMap tmK, DecWs ws, int W, int chunk,
                     int nl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * DS_WARPS + warp;
  const int T = (a.num_q + 3) / 4;
  const int tile = gw / W, wc = gw % W;
  if (tile >= T) return;  // the whole CTA (W is a multiple of DS_WARPS)
  const bool cta_merge = nl != W;

  const uint32_t stage0 = smem_addr(smem) + warp * (DS_NST * DS_PAGE);
  u64* buf = reinterpret_cast<u64*>(smem + DecSmem::STAGES) + warp * 4 * DS_CAP;
  u64* mlist = reinterpret_cast<u64*>(smem + DecSmem::STAGES + DecSmem::BUF);  // [warp][row][16]
  u64* mbound = mlist + DS_WARPS * 4 * DS_KW;                                  // [warp][row]
  int* pid = reinterpret_cast<int*>(mbound + DS_WARPS * 4) + warp * DS_MAXPG;
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<int*>(mbound + DS_WARPS * 4) +
                                              DS_WARPS * DS_MAXPG) + warp * DS_NST;
  if (lane == 0) {
    for (int s = 0; s < DS_NST; ++s) mbar_init(&bar[s], 1);
    mbar_fence_init();
  }
  // a (warp chunk, row) list and bound: straight to the workspace, or to the CTA merge
  auto put_list = [&](int r, u64 key, bool half_owner, u64 bound) {
    if (cta_merge) {
      if (half_owner) mlist[(warp * 4 + r) * DS_KW + (lane & 15)] = key;
      if (lane == 0) mbound[warp * 4 + r] = bound;
    } else {
      const long long row = (long long)tile * 4 + r;
      if (half_owner) ws.lists[(row * nl + wc) * DS_KW + (lane & 15)] = key;
      if (lane == 0) ws.bounds[row * pad2(nl) + wc] = bound;
    }
  };

  // the tile's rows: lanes 0..3 validate, everyone gets all four
  int seq_l = -1, lim_l = -1;
  if (lane < 4 && tile * 4 + lane < a.num_q) {
    int sq = -1;
    const int l = row_limit(a, tile * 4 + lane, &sq);
    if (l >= 0) {
      seq_l = sq;
      lim_l = l;
    }
  }
  int rseq[4], rlim[4];
  uint32_t done = 0;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    rseq[r] = __shfl_sync(0xffffffffu, seq_l, r);
    rlim[r] = __shfl_sync(0xffffffffu, lim_l, r);
    if (rseq[r] < 0) done |= 1u << r;
  }
#pragma unroll
  for (int r = 0; r < 4; ++r)  // invalid or absent rows: empty lists
    if (done >> r & 1u) put_list(r, 0ull, (lane >> 4) == 0, 0ull);
  __syncwarp();

  // ldmatrix: this lane's row (block) and the 16-byte chunk offsets of its four k-steps per half
  const int lblk = (lane & 7) + ((lane >> 4) << 3);
  uint32_t koff[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) koff[q] = lblk * 128 + (((q * 2 + ((lane >> 3) & 1)) ^ (lblk & 7)) << 4);
  const int rr = (lane >> 2) & 3;  // this lane's query row (C rows lane/4 and lane/4 + 8)
  const int hlo = lane >> 4;       // and heads hlo, hlo + 2
  const int c4 = lane & 3;
  const unsigned rowmask = 0x000F000Fu << (4 * rr);
  const unsigned lt = (1u << lane) - 1u;
  int base = 0;                    // pages consumed by this warp so far (ring position)
  bool aborted = false;

  while (done != 0xFu && !aborted) {
    const int r0 = __ffs(~done & 0xFu) - 1;
    const int seg = __shfl_sync(0xffffffffu, seq_l, r0);
    uint32_t mrows = 0;
    int nbmax = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if (!(done >> r & 1u) && rseq[r] == seg) {
        mrows |= 1u << r;
        nbmax = max(nbmax, rlim[r]);
      }
    done |= mrows;
    const bool mine = (mrows >> rr) & 1u;
    const int lim_rr = __shfl_sync(0xffffffffu, lim_l, rr);
    const int lim = mine ? lim_rr : -1;
    const int p0 = wc * chunk;
    const int np = max(0, min(p0 + chunk, (nbmax + 15) / 16) - p0);

    for (int i = lane; i < np; i += 32) {
      int pg = a.page_table[(long long)seg * a.max_pages + p0 + i];
      if (pg < 0 || pg >= a.num_pages) {
        flag_error(a.err, QSA_DEVERR_PAGE);
        pg = -1;
      }
      pid[i] = pg;
    }
    __syncwarp();
    auto issue = [&](int i) {  // lane 0 only
      const int s = (base + i) % DS_NST;
      const int pg = pid[i];
      if (pg >= 0) {
        // the stage's earlier ldmatrix reads (generic proxy) before the TMA writes (async proxy)
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        mbar_arrive_expect_tx(&bar[s], DS_PAGE);
        const uint64_t pol = l2_evict_first_policy();
        tma2d_hint(stage0 + s * DS_PAGE, &tmK, 0, pg * 16, &bar[s], pol);
        tma2d_hint(stage0 + s * DS_PAGE + DS_PAGE / 2, &tmK, 64, pg * 16, &bar[s], pol);
      } else {
        mbar_arrive(&bar[s]);  // no data: the page's blocks are masked below
      }
    };
    if (lane == 0)
      for (int i = 0; i < min(np, DS_NST); ++i) issue(i);

    // query fragments of this segment's rows (zeros for the tile's other rows)
    uint32_t afr[8][4];
    float wa = 0.f, wb = 0.f;
    {
      const int row = tile * 4 + rr;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.idx_q + ((long long)row * kHi + hlo) * 128);
      const uint32_t* q2 = q0 + 2 * 64;  // head hlo + 2
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        afr[ks][0] = mine ? q0[ks * 8 + c4] : 0u;
        afr[ks][1] = mine ? q2[ks * 8 + c4] : 0u;
        afr[ks][2] = mine ? q0[ks * 8 + c4 + 4] : 0u;
        afr[ks][3] = mine ? q2[ks * 8 + c4 + 4] : 0u;
      }
      if (mine) {
        wa = __bfloat162float(a.idx_w[(long long)row * kHi + hlo]);
        wb = __bfloat162float(a.idx_w[(long long)row * kHi + hlo + 2]);
      }
    }

    int cnt = 0;  // keys in this lane's row buffer
    // candidate blocks of this lane's row in the chunk (an invalid page, already flagged, counts too)
    const int nvalid = mine ? max(0, min(lim, (p0 + np) * 16) - p0 * 16) : 0;
    uint32_t thr_hi = 0, thr_lo = 0;  // this lane's row threshold (its list's 16th key)
    // top2[p]: the lists of rows 2p (lanes 0-15) and 2p+1 (lanes 16-31), rank = lane & 15
    u64 top2[2] = {0ull, 0ull};
    auto merge_pair = [&](const int p) {  // fold the buffers of rows 2p, 2p+1 into their lists
      const int c0 = __shfl_sync(0xffffffffu, cnt, 8 * p);
      const int c1 = __shfl_sync(0xffffffffu, cnt, 8 * p + 4);
      const int myr = 2 * p + (lane >> 4);
      const int myc = (lane >> 4) ? c1 : c0;
      u64 t = top2[p];
      for (int g = 0; g < max(c0, c1); g += 16) {
        const int idx = g + (lane & 15);
        t = half_merge16(t, idx < myc ? buf[myr * DS_CAP + idx] : 0ull);
      }
      top2[p] = t;
      const u64 t0 = __shfl_sync(0xffffffffu, t, 15), t1 = __shfl_sync(0xffffffffu, t, 31);
      if (rr == 2 * p || rr == 2 * p + 1) {
        const u64 tv = rr == 2 * p ? t0 : t1;
        cnt = 0;
        thr_hi = (uint32_t)(tv >> 32);
        thr_lo = (uint32_t)tv;
      }
      __syncwarp();
    };
    int i = 0;
    for (; i < np; ++i) {
      const int s = (base + i) % DS_NST;
      if (!mbar_wait(&bar[s], (uint32_t)((base + i) / DS_NST) & 1u, a.err)) {
        aborted = true;
        break;
      }
      const uint32_t st = stage0 + s * DS_PAGE;
      float acc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t bfr[4];
        ldsm_x4(bfr, st + (ks >> 2) * (DS_PAGE / 2) + koff[ks & 3]);
        mma_bf16_16816(acc[0], afr[ks], bfr[0], bfr[1]);
        mma_bf16_16816(acc[1], afr[ks], bfr[2], bfr[3]);
      }
      const bool page_ok = pid[i] >= 0;
      __syncwarp();
      if (lane == 0 && i + DS_NST < np) issue(i + DS_NST);  // the stage's reads are done
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float p0v = fmaf(wb, fmaxf(acc[nt][2], 0.f), wa * fmaxf(acc[nt][0], 0.f));
        const float p1v = fmaf(wb, fmaxf(acc[nt][3], 0.f), wa * fmaxf(acc[nt][1], 0.f));
        const float send = hlo ? p0v : p1v;
        const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
        const float sc = hlo ? p1v + recv : p0v + recv;
        const int b = (p0 + i) * 16 + nt * 8 + 2 * c4 + hlo;
        // key = ordered score : (0xFFFFFFFF - block); compared with the threshold in two halves
        const uint32_t ord = f32_to_ordered(__fadd_rn(sc, 0.0f));
        const uint32_t lo = 0xFFFFFFFFu - (uint32_t)b;
        const bool pass = page_ok && b < lim && (ord > thr_hi || (ord == thr_hi && lo > thr_lo));
        const unsigned bal = __ballot_sync(0xffffffffu, pass);
        if (pass) buf[rr * DS_CAP + cnt + __popc(bal & rowmask & lt)] = ((u64)ord << 32) | lo;
        cnt += __popc(bal & rowmask);
      }
      __syncwarp();
      {  // a buffer that the next page could overflow is folded into its list
        const unsigned near_full = __ballot_sync(0xffffffffu, cnt > DS_CAP - 16);
        if (near_full & 0x00FF00FFu) merge_pair(0);
        if (near_full & 0xFF00FF00u) merge_pair(1);
      }
    }
    if (aborted) {
      // a page never arrived (reported as QSA_DEVERR_TIMEOUT): wait, bounded, for the copies
      // still in flight into this warp's ring; the maximal bound makes the merge hand the
      // tile's rows to the exact kernel
      for (int j = i; j < min(np, i + DS_NST); ++j)
        mbar_wait(&bar[(base + j) % DS_NST], (uint32_t)((base + j) / DS_NST) & 1u, a.err);
#pragma unroll
      for (int r = 0; r < 4; ++r) put_list(r, 0ull, (lane >> 4) == 0, ~0ull);
      break;
    }
    base += np;
    merge_pair(0);
    merge_pair(1);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (!(mrows >> r & 1u)) continue;
      const u64 t = top2[r >> 1];
      // keys were dropped iff the chunk had more candidates than the list holds; they are all
      // below the list's 16th key
      const bool dropped = __shfl_sync(0xffffffffu, nvalid, 4 * r) > DS_KW;
      const u64 kth = __shfl_sync(0xffffffffu, t, (r & 1) ? 31 : 15);
      put_list(r, t, (lane >> 4) == (r & 1), dropped ? kth : 0ull);
    }
    __syncwarp();
  }

  if (!cta_merge) return;
  // CTA merge: warp r (< 4) folds the DS_WARPS lists of row r into one list of DS_KC keys
  __syncthreads();
  const int r = warp;
  if (r >= 4 || tile * 4 + r >= a.num_q) return;
  u64 top = 0, bound = 0;
  int nz = 0;
  for (int w = 0; w < DS_WARPS; w += 2) {
    const u64 v = mlist[((w + (lane >> 4)) * 4 + r) * DS_KW + (lane & 15)];
    nz += __popc(__ballot_sync(0xffffffffu, v != 0ull));
    top = warp_fold_two16(top, v);
  }
  for (int w = 0; w < DS_WARPS; ++w) bound = mbound[w * 4 + r] > bound ? mbound[w * 4 + r] : bound;
  const u64 kth = __shfl_sync(0xffffffffu, top, 31);
  if (nz > DS_KC && kth > bound) bound = kth;  // the CTA merge itself dropped keys below kth
  const long long row = (long long)tile * 4 + r;
  const int cidx = wc / DS_WARPS;
  ws.lists[(row * nl + cidx) * DS_KC + lane] = top;
  if (lane == 0) ws.bounds[row * pad2(nl) + cidx] = bound;
}

// ------------------------------------------------------------------ merge (one CTA per row)

constexpr int DM_CAND = 512;  // keys of the boundary histogram bin ranked directly

struct MergeSmem {
  static constexpr int KEYS = DM_MAXU * 8;
  static constexpr int BOUNDS = DS_MAXW * 8;
  static constexpr int HIST = 2048 * 4;
  static constexpr int CAND = DM_CAND * 8;
  static constexpr int LISTS = 2 * DS_MAXW * 4;  // selected count and output offset per list
  static constexpr int TAIL = 640;  // reductions, barrier, scan totals, selection scalars
  static constexpr int TOTAL = KEYS + BOUNDS + HIST + CAND + LISTS + TAIL;
};

// Exclusive prefix sum over the CTA (DM_THREADS threads); wsum: 32 words of shared memory.
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = lane < DM_THREADS / 32 ? wsum[lane] : 0u;
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += x;
    }
    if (lane < DM_THREADS / 32) wsum[lane] = ti - t;
  }
  __syncthreads();
  const uint32_t r = wsum[warp] + incl - v;
  __syncthreads();
  return r;
}

__device__ __forceinline__ u64 cta_min_u64(u64 v, u64* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const u64 x = __shfl_xor_sync(0xffffffffu, v, o);
    v = x < v ? x : v;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  u64 m = ~0ull;
  for (int w = 0; w < DM_THREADS / 32; ++w) m = red[w] < m ? red[w] : m;
  __syncthreads();
  return m;
}

__device__ __forceinline__ u64 cta_max_u64(u64 v, u64* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const u64 x = __shfl_xor_sync(0xffffffffu, v, o);
    v = x > v ? x : v;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  u64 m = 0;
  for (int w = 0; w < DM_THREADS / 32; ++w) m = red[w] > m ? red[w] : m;
  __syncthreads();
  return m;
}

// The need-th largest of n unique keys in shared memory (1 <= need <= n), by the whole CTA:
// MSB-first radix select with 11-bit digits starting at the highest bit where the keys differ.
__device__ u64 cta_kth_largest(const u64* keys, int n, int need, uint32_t* hist, u64* red,
                               uint32_t* wsum, uint32_t* sel3) {
  const int tid = threadIdx.x;
  u64 lo = ~0ull, hi = 0ull;
  for (int i = tid; i < n; i += DM_THREADS) {
    const u64 k = keys[i];
    lo = k < lo ? k : lo;
    hi = k > hi ? k : hi;
  }
  lo = cta_min_u64(lo, red);
  hi = cta_max_u64(hi, red);
  if (need == n) return lo;
  if (need == 1) return hi;
  int top = 63 - __clzll((long long)(lo ^ hi));
  u64 prefix = 0, mask = 0;
  if (top < 63) {
    mask = ~((2ull << top) - 1ull);
    prefix = hi & mask;
  }
  uint32_t remaining = (uint32_t)need;
  for (;;) {
    const int width = top + 1 < 11 ? top + 1 : 11;
    const int shift = top + 1 - width;
    const int nb = 1 << width;
    for (int i = tid; i < nb; i += DM_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += DM_THREADS) {
      const u64 k = keys[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(uint32_t)(k >> shift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    const int per = (nb + DM_THREADS - 1) / DM_THREADS;  // bins per thread, counted from the top
    uint32_t tot = 0;
    for (int j = 0; j < per; ++j) {
      const int bin = nb - 1 - (tid * per + j);
      if (bin >= 0) tot += hist[bin];
    }
    const uint32_t excl = cta_excl_scan(tot, wsum);
    if (excl < remaining && remaining <= excl + tot) {
      uint32_t acc = excl;
      for (int j = 0; j < per; ++j) {
        const int bin = nb - 1 - (tid * per + j);
        const uint32_t c = hist[bin];
        if (acc + c >= remaining) {
          sel3[0] = (uint32_t)bin;
          sel3[1] = acc;
          sel3[2] = c;
          break;
        }
        acc += c;
      }
    }
    __syncthreads();
    const uint32_t digit = sel3[0], above = sel3[1], cnt_at = sel3[2];
    __syncthreads();
    remaining -= above;
    prefix |= (u64)digit << shift;
    mask |= (u64)(nb - 1) << shift;
    if (shift == 0) return prefix;
    if (cnt_at == remaining) {  // every key under this prefix is kept: the answer is their min
      u64 m = ~0ull;
      for (int i = tid; i < n; i += DM_THREADS) {
        const u64 k = keys[i];
        if ((k & mask) == prefix && k < m) m = k;
      }
      return cta_min_u64(m, red);
    }
    top = shift - 1;
  }
}

// One CTA per query row.  The row's lists come in block order (list l covers a block range below
// list l+1's) and each is sorted by key, so the need keys >= tau are a prefix of every list: the
// output is the lists' prefixes in list order, each put in block order by a warp-level rank.
__global__ void __launch_bounds__(DM_THREADS)
    dec_merge_kernel(ScoreArgs a, DecWs ws, int nl, int lk) {
  extern __shared__ __align__(128) uint8_t smem[];
  u64* keys = reinterpret_cast<u64*>(smem);
  u64* bnds = reinterpret_cast<u64*>(smem + MergeSmem::KEYS);
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + MergeSmem::KEYS + MergeSmem::BOUNDS);
  u64* cand = reinterpret_cast<u64*>(smem + MergeSmem::KEYS + MergeSmem::BOUNDS + MergeSmem::HIST);
  int* lcnt = reinterpret_cast<int*>(smem + MergeSmem::KEYS + MergeSmem::BOUNDS + MergeSmem::HIST +
                                     MergeSmem::CAND);
  int* loff = lcnt + DS_MAXW;
  uint8_t* tail = reinterpret_cast<uint8_t*>(loff + DS_MAXW);
  u64* red = reinterpret_cast<u64*>(tail);                    // [3][16] per-warp min, max, bound
  uint32_t* redn = reinterpret_cast<uint32_t*>(tail + 384);  // [16] per-warp kept counts
  uint64_t* bar = reinterpret_cast<uint64_t*>(tail + 448);
  uint32_t* wsum = reinterpret_cast<uint32_t*>(tail + 456);  // [16] scan totals
  uint32_t* sel3 = reinterpret_cast<uint32_t*>(tail + 520);  // digit, above, count, n in bin
  u64* s_tau = reinterpret_cast<u64*>(tail + 536);

  const int row = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NW = DM_THREADS / 32;
  const int seq = a.q_seq[row], pos = a.q_pos[row];
  const bool ok = seq >= 0 && seq < a.batch && pos >= 0 && pos / 64 < a.max_pages && pos <= a.max_pos;
  if (!ok) {  // already flagged by the score kernel
    if (warp == 0) write_empty_selection(row, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
    if (tid == 0) ws.redo[row] = 0;
    return;
  }
  const int lim = pos / 4;
  const int need = min(a.topk, lim);
  int32_t* srow = a.sel + (long long)row * a.sel_stride;
  float* crow = a.sel_scores ? a.sel_scores + (long long)row * a.sel_stride : nullptr;
  // the tail block and the padding after the need selected blocks
  for (int i = need + tid; i < a.sel_stride; i += DM_THREADS) {
    srow[i] = i == need ? lim : -1;
    if (crow) crow[i] = i == need ? __int_as_float(0x7f800000) : __int_as_float(0x7fc00000);
  }
  if (need == 0) {
    if (tid == 0) {
      a.n_sel[row] = 1;
      ws.redo[row] = 0;
    }
    return;
  }

  // the row's nl lists (zero-padded) and their bounds, one bulk copy each
  const int nlp = pad2(nl);
  const int U = nl * lk;
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)(U * 8 + nlp * 8));
    bulk_g2s(smem_addr(keys), ws.lists + (long long)row * U, (uint32_t)(U * 8), bar);
    bulk_g2s(smem_addr(bnds), ws.bounds + (long long)row * nlp, (uint32_t)(nlp * 8), bar);
  }
  const bool arrived = mbar_wait(bar, 0, a.err);
  if (!__syncthreads_and(arrived)) {  // reported as a timeout; the exact kernel redoes the row
    if (tid == 0) {
      ws.redo[row] = 1;
      mbar_wait(bar, 0, a.err);  // and the copies still in flight land first (bounded)
    }
    return;
  }

  // one pass: kept keys, smallest kept and largest key, and the largest bound (every key a list
  // dropped lies below its bound), reduced per warp and then by every thread from 16 entries
  uint32_t nk = 0;
  u64 lo = ~0ull, hi = 0ull, mb = 0ull;
  for (int i = tid; i < U; i += DM_THREADS) {
    const u64 k = keys[i];
    if (k) {
      ++nk;
      lo = k < lo ? k : lo;
      hi = k > hi ? k : hi;
    }
  }
  for (int i = tid; i < nl; i += DM_THREADS) mb = bnds[i] > mb ? bnds[i] : mb;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nk += __shfl_xor_sync(0xffffffffu, nk, o);
    const u64 x = __shfl_xor_sync(0xffffffffu, lo, o), y = __shfl_xor_sync(0xffffffffu, hi, o),
              z = __shfl_xor_sync(0xffffffffu, mb, o);
    lo = x < lo ? x : lo;
    hi = y > hi ? y : hi;
    mb = z > mb ? z : mb;
  }
  if (lane == 0) {
    red[warp] = lo;
    red[16 + warp] = hi;
    red[32 + warp] = mb;
    redn[warp] = nk;
  }
  __syncthreads();
  // every warp reduces the NW per-warp entries itself: one entry per lane, then shuffles
  static_assert(NW <= 32, "one per-warp entry per lane");
  nk = lane < NW ? redn[lane] : 0u;
  lo = lane < NW ? red[lane] : ~0ull;
  hi = lane < NW ? red[16 + lane] : 0ull;
  mb = lane < NW ? red[32 + lane] : 0ull;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nk += __shfl_xor_sync(0xffffffffu, nk, o);
    const u64 x = __shfl_xor_sync(0xffffffffu, lo, o), y = __shfl_xor_sync(0xffffffffu, hi, o),
              z = __shfl_xor_sync(0xffffffffu, mb, o);
    lo = x < lo ? x : lo;
    hi = y > hi ? y : hi;
    mb = z > mb ? z : mb;
  }
  if ((int)nk < need) {  // lists dropped too much: the exact kernel redoes the row
    if (tid == 0) ws.redo[row] = 1;
    return;
  }

  // tau = the need-th largest kept key: one CTA histogram of 11 bits below the highest bit where
  // the kept keys differ, then the few keys of the boundary bin are ranked directly
  u64 tau;
  if ((int)nk == need) {
    tau = lo;
  } else {
    const int top = 63 - __clzll((long long)(lo ^ hi));
    const int width = top + 1 < 11 ? top + 1 : 11;
    const int shift = top + 1 - width;
    const uint32_t nb = 1u << width;
    const u64 hmask = top < 63 ? ~((2ull << top) - 1ull) : 0ull;  // bits every kept key shares
    const u64 prefix = hi & hmask;
    for (uint32_t i = tid; i < nb; i += DM_THREADS) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < U; i += DM_THREADS) {
      const u64 k = keys[i];
      if (k && (k & hmask) == prefix) atomicAdd(&hist[(uint32_t)(k >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    const int per = (int)(nb + DM_THREADS - 1) / DM_THREADS;  // bins per thread from the top
    uint32_t tot = 0;
    for (int j = 0; j < per; ++j) {
      const int bin = (int)nb - 1 - (tid * per + j);
      if (bin >= 0) tot += hist[bin];
    }
    const uint32_t excl = cta_excl_scan(tot, wsum);
    if (excl < (uint32_t)need && (uint32_t)need <= excl + tot) {
      uint32_t acc = excl;
      for (int j = 0; j < per; ++j) {
        const int bin = (int)nb - 1 - (tid * per + j);
        const uint32_t c = hist[bin];
        if (acc + c >= (uint32_t)need) {
          sel3[0] = (uint32_t)bin;
          sel3[1] = acc;  // kept keys in higher bins
          sel3[2] = c;
          break;
        }
        acc += c;
      }
    }
    if (tid == 0) sel3[3] = 0;
    __syncthreads();
    const uint32_t digit = sel3[0], above = sel3[1], inbin = sel3[2];
    if (inbin <= (uint32_t)DM_THREADS) {
      // the boundary bin's keys, each ranked by counting the larger ones (keys are unique)
      const u64 bmask = hmask | ((u64)(nb - 1) << shift);
      const u64 bpre = prefix | ((u64)digit << shift);
      for (int i = tid; i < U; i += DM_THREADS) {
        const u64 k = keys[i];
        if (k && (k & bmask) == bpre) cand[atomicAdd(&sel3[3], 1u)] = k;
      }
      __syncthreads();
      if (tid < (int)inbin) {
        const u64 k = cand[tid];
        uint32_t r = 0;
        for (uint32_t j = 0; j < inbin; ++j) r += cand[j] > k;
        if (r == (uint32_t)need - above - 1u) *s_tau = k;
      }
      __syncthreads();
      tau = *s_tau;
    } else {  // a crowded bin: the full CTA radix select
      tau = cta_kth_largest(keys, U, need, hist, red, wsum, sel3);
    }
  }
  if (mb > tau) {  // a dropped key could beat tau: the exact kernel redoes the row
    if (tid == 0) ws.redo[row] = 1;
    return;
  }

  // keys >= tau per list (a prefix: lists are sorted by key), then each list's output offset
  for (int w = warp; w < nl; w += NW) {
    const bool sel = lane < lk && keys[w * lk + lane] >= tau;
    const int c = __popc(__ballot_sync(0xffffffffu, sel));
    if (lane == 0) lcnt[w] = c;
  }
  __syncthreads();
  {
    int c0 = 2 * tid < nl ? lcnt[2 * tid] : 0, c1 = 2 * tid + 1 < nl ? lcnt[2 * tid + 1] : 0;
    const uint32_t ex = cta_excl_scan((uint32_t)(c0 + c1), wsum);
    if (2 * tid < nl) loff[2 * tid] = (int)ex;
    if (2 * tid + 1 < nl) loff[2 * tid + 1] = (int)ex + c0;
  }
  __syncthreads();
  // each list's selected keys in block order: rank by comparison within the prefix
  for (int w = warp; w < nl; w += NW) {
    const int c = lcnt[w];
    if (c == 0) continue;
    const u64 k = lane < c ? keys[w * lk + lane] : 0ull;
    const uint32_t b = lane < c ? key_block(k) : 0xFFFFFFFFu;
    int r = 0;
    for (int j = 0; j < c; ++j) r += __shfl_sync(0xffffffffu, b, j) < b;
    if (lane < c) {
      const int o = loff[w] + r;
      srow[o] = (int32_t)b;
      if (crow) crow[o] = key_score(k);
    }
  }
  if (tid == 0) {
    a.n_sel[row] = need + 1;
    ws.redo[row] = 0;
  }
}

}  // namespace

bool score_dec_plan_ok(const Geometry& g) {
  DecPlan p;
  return g.Di == 128 && g.topk <= 512 && dec_plan(g, &p);
}

size_t score_dec_redo_offset(const Geometry& g) {
  DecPlan p;
  if (!dec_plan(g, &p)) return 0;
  return stream_region(g) + r256((size_t)p.T * 4 * p.nl * p.lk * 8) + r256((size_t)p.T * 4 * pad2(p.nl) * 8);
}

size_t score_dec_workspace_bytes(const Geometry& g) {
  DecPlan p;
  if (!dec_plan(g, &p)) return 0;
  return stream_region(g) + r256((size_t)p.T * 4 * p.nl * p.lk * 8) +
         r256((size_t)p.T * 4 * pad2(p.nl) * 8) + r256((size_t)g.num_q * 4);
}

cudaError_t launch_score_dec(const ScoreArgs& a, const Geometry& g, void* ws, int32_t** redo_out,
                             cudaStream_t s) {
  auto enc = tmap_encode_fn();
  DecPlan p;
  if (!enc || !dec_plan(g, &p)) return cudaErrorNotSupported;
  const DecWs w = carve_dec(g, p, ws);
  *redo_out = w.redo;
  CUtensorMap tmK;
  {
    cuuint64_t dims[2] = {128, (cuuint64_t)g.num_pages * 16};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(a.kcomp), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = set_smem_once(dec_score_kernel, DecSmem::TOTAL);
  if (e != cudaSuccess) return e;
  e = set_smem_once(dec_merge_kernel, MergeSmem::TOTAL);
  if (e != cudaSuccess) return e;
  const int warps = p.T * p.W;
  dec_score_kernel<<<warps / DS_WARPS, DS_THREADS, DecSmem::TOTAL, s>>>(a, tmK, w, p.W, p.chunk, p.nl);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dec_merge_kernel<<<g.num_q, DM_THREADS, MergeSmem::TOTAL, s>>>(a, w, p.nl, p.lk);
  return cudaGetLastError();
}

}  // namespace qsa
