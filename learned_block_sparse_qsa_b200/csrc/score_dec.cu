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
// more than 16 of the row's top 512 to fail (expected ~1); a row that fails is flagged, and the
// same CTA then selects exactly over every candidate of the row (exact_row_body), so the result
// never depends on the split.
#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"
#include "select.cuh"
#include "attn_sw.cuh"

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

template <int NW>
struct DecSmemT {
  static constexpr int STAGES = NW * DS_NST * DS_PAGE;  // first, 1024-byte aligned
  static constexpr int BUF = NW * 4 * DS_CAP * 8;
  static constexpr int MLIST = NW * 4 * DS_KW * 8;      // warp lists for the CTA merge
  static constexpr int MBOUND = NW * 4 * 8;
  static constexpr int PID = NW * DS_MAXPG * 4;
  static constexpr int BAR = NW * DS_NST * 8;
  static constexpr int TOTAL = STAGES + BUF + MLIST + MBOUND + PID + BAR + 1024;  // + alignment
};
using DecSmem = DecSmemT<DS_WARPS>;
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
// nw: warps per CTA; resident_warps: warps the GPU runs at once (all of them stream together).
bool dec_plan_nw(const Geometry& g, int nw, long long resident_warps, DecPlan* p) {
  p->T = (g.num_q + 3) / 4;
  const long long pages = ((long long)g.max_pos / 4 + 15) / 16;  // candidates are b < t/4
  const long long P = pages > 0 ? pages : 1;
  long long W = (resident_warps + p->T - 1) / p->T;
  W = W < DS_MINW ? DS_MINW : (W > DS_MAXW ? DS_MAXW : W);
  if (W > P) W = P;
  long long chunk = (P + W - 1) / W;
  if (chunk > DS_MAXPG) chunk = DS_MAXPG;
  W = (P + chunk - 1) / chunk;
  W = (W + nw - 1) / nw * nw;  // trailing chunks may be empty
  if (W > DS_MAXW) return false;
  p->W = (int)W;
  p->chunk = (int)chunk;
  const bool merge = W >= DS_CTA_MERGE_W;
  p->nl = merge ? p->W / nw : p->W;
  p->lk = merge ? DS_KC : DS_KW;
  return true;
}
bool dec_plan(const Geometry& g, DecPlan* p) {
  return dec_plan_nw(g, DS_WARPS, (long long)DS_CTAS * num_sms() * DS_WARPS, p);
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

// A region the size of the exact streaming kernel's candidate buffers sits at the workspace base
// (unused by the decode forms: their exact path keeps its keys in a region of its own); the
// lists, bounds and flags follow it.
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

// Optional wait of the warps whose pages hold blocks compressed earlier in the same launch (the
// fused decode step): they wait for `*ctr >= target` before streaming those pages.
struct NewBlockWait {
  const int* ctr = nullptr;
  int target = 0;
  const int32_t* new_seq = nullptr;
  const int32_t* new_pos = nullptr;
  int n_groups = 0;
};

// The streaming part of the decode indexer for virtual CTA `vblock` of NW warps (all threads of
// the calling block take part).  smem_raw: DecSmemT<NW>::TOTAL bytes.
// ltid: the thread's index within the NW warps running the body (warp-aligned); bar_id: the named
// barrier over those NW * 32 threads (0: the whole block is exactly those threads).
template <int NW>
__device__ __forceinline__ void dec_score_body(const ScoreArgs& a, const CUtensorMap* tmK, const DecWs& ws,
                                               int W, int chunk, int nl, int vblock, uint8_t* smem_raw,
                                               const NewBlockWait& nbw, const int ltid = threadIdx.x,
                                               const int bar_id = 0) {
  using DecSmem = DecSmemT<NW>;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = ltid >> 5, lane = ltid & 31;
  const int gw = vblock * NW + warp;
  const int T = (a.num_q + 3) / 4;
  const int tile = gw / W, wc = gw % W;
  if (tile >= T) return;  // the whole CTA (W is a multiple of NW)
  const bool cta_merge = nl != W;

  const uint32_t stage0 = smem_addr(smem) + warp * (DS_NST * DS_PAGE);
  u64* buf = reinterpret_cast<u64*>(smem + DecSmem::STAGES) + warp * 4 * DS_CAP;
  u64* mlist = reinterpret_cast<u64*>(smem + DecSmem::STAGES + DecSmem::BUF);  // [warp][row][16]
  u64* mbound = mlist + NW * 4 * DS_KW;                                  // [warp][row]
  int* pid = reinterpret_cast<int*>(mbound + NW * 4) + warp * DS_MAXPG;
  uint64_t* bar = reinterpret_cast<uint64_t*>(reinterpret_cast<int*>(mbound + NW * 4) +
                                              NW * DS_MAXPG) + warp * DS_NST;
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
    if (nbw.ctr && lane == 0) {  // pages holding blocks compressed earlier in this launch
      bool hit = false;
      for (int j = 0; j < nbw.n_groups && !hit; ++j) {
        const int bp = nbw.new_pos[4 * j] / 64;
        hit = nbw.new_seq[4 * j] == seg && bp >= p0 && bp < p0 + np;
      }
      if (hit) {
        const volatile int* c = nbw.ctr;
        const long long t0 = clock64();
        while (*c < nbw.target) {
          if (clock64() - t0 > kWaitLimitCycles) {
            flag_error(a.err, QSA_DEVERR_TIMEOUT);
            break;
          }
        }
        __threadfence();
        asm volatile("fence.proxy.async.global;\n" ::: "memory");
      }
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
        tma2d_hint(stage0 + s * DS_PAGE, tmK, 0, pg * 16, &bar[s], pol);
        tma2d_hint(stage0 + s * DS_PAGE + DS_PAGE / 2, tmK, 64, pg * 16, &bar[s], pol);
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
      // tile's rows to the exact path
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
  // CTA merge: warp r (< 4) folds the NW lists of row r into one list of DS_KC keys
  if (bar_id == 0) __syncthreads();
  else asm volatile("bar.sync %0, %1;\n" ::"r"(bar_id), "n"(NW * 32) : "memory");
  const int r = warp;
  if (r >= 4 || tile * 4 + r >= a.num_q) return;
  u64 top = 0, bound = 0;
  int nz = 0;
  for (int w = 0; w < NW; w += 2) {
    const u64 v = mlist[((w + (lane >> 4)) * 4 + r) * DS_KW + (lane & 15)];
    nz += __popc(__ballot_sync(0xffffffffu, v != 0ull));
    top = warp_fold_two16(top, v);
  }
  for (int w = 0; w < NW; ++w) bound = mbound[w * 4 + r] > bound ? mbound[w * 4 + r] : bound;
  const u64 kth = __shfl_sync(0xffffffffu, top, 31);
  if (nz > DS_KC && kth > bound) bound = kth;  // the CTA merge itself dropped keys below kth
  const long long row = (long long)tile * 4 + r;
  const int cidx = wc / NW;
  ws.lists[(row * nl + cidx) * DS_KC + lane] = top;
  if (lane == 0) ws.bounds[row * pad2(nl) + cidx] = bound;
}

__global__ void __launch_bounds__(DS_THREADS, DS_CTAS)
    dec_score_kernel(ScoreArgs a, const __grid_constant__ CUtensorMap tmK, DecWs ws, int W, int chunk,
                     int nl) {
  extern __shared__ uint8_t smem_raw[];
  chain_wait();
  // No early release: the merge's 16 CTAs, scheduled early, would take the first SMs that free
  // up, two to an SM; launched at this grid's exit they spread out (C5 graph 97.6 against
  // 99.6 us with the release).
  dec_score_body<DS_WARPS>(a, &tmK, ws, W, chunk, nl, blockIdx.x, smem_raw, NewBlockWait{});
}

// ------------------------------------------------------------------ merge (one CTA per row)

constexpr int DM_CAND = 512;        // capacity of the boundary-bin key list
constexpr int DM_RANK_DIRECT = 64;  // a boundary bin this small is ranked by direct comparison;
                                    // a larger one costs O(n^2) there and is refined instead

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

// Radix-select continuation: among the keys k with (k & mask) == prefix -- the bits above bit
// `top` already decided -- the `remaining`-th largest, by 11-bit digits from bit `top` down.
__device__ u64 cta_kth_refine(const u64* keys, int n, uint32_t remaining, u64 prefix, u64 mask, int top,
                              uint32_t* hist, u64* red, uint32_t* wsum, uint32_t* sel3) {
  const int tid = threadIdx.x;
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
  const int top = 63 - __clzll((long long)(lo ^ hi));
  u64 prefix = 0, mask = 0;
  if (top < 63) {
    mask = ~((2ull << top) - 1ull);
    prefix = hi & mask;
  }
  return cta_kth_refine(keys, n, (uint32_t)need, prefix, mask, top, hist, red, wsum, sel3);
}

// One CTA per query row.  The row's lists come in block order (list l covers a block range below
// list l+1's) and each is sorted by key, so the need keys >= tau are a prefix of every list: the
// output is the lists' prefixes in list order, each put in block order by a warp-level rank.
// The merge of query row `row` by all DM_THREADS threads of the calling block; smem:
// MergeSmem::TOTAL bytes, 128-byte aligned.  A row it cannot settle gets ws.redo[row] = 1.
__device__ __forceinline__ void dec_merge_body(const ScoreArgs& a, const DecWs& ws, int nl, int lk,
                                               const int row, uint8_t* smem) {
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

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NW = DM_THREADS / 32;
  if (tid == 0) {  // initialised on every path, so that a caller can invalidate it afterwards
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
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
    mbar_arrive_expect_tx(bar, (uint32_t)(U * 8 + nlp * 8));
    bulk_g2s(smem_addr(keys), ws.lists + (long long)row * U, (uint32_t)(U * 8), bar);
    bulk_g2s(smem_addr(bnds), ws.bounds + (long long)row * nlp, (uint32_t)(nlp * 8), bar);
  }
  const bool arrived = mbar_wait(bar, 0, a.err);
  if (!__syncthreads_and(arrived)) {  // reported as a timeout; the exact path redoes the row
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
  if ((int)nk < need) {  // lists dropped too much: the exact path redoes the row
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
    if (inbin <= (uint32_t)DM_RANK_DIRECT) {
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
    } else {  // a crowded bin: refine by the next digits below it
      __syncthreads();
      const u64 bmask = hmask | ((u64)(nb - 1) << shift);
      const u64 bpre = prefix | ((u64)digit << shift);
      tau = shift == 0 ? bpre
                       : cta_kth_refine(keys, U, (uint32_t)need - above, bpre, bmask, shift - 1, hist, red,
                                        wsum, sel3);
    }
  }
  if (mb > tau) {  // a dropped key could beat tau: the exact path redoes the row
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


// ------------------------------------------------------------------ exact path for one row
// The row's every candidate score on CUDA cores (4 heads x 128 dims per block), as 64-bit keys in
// `keys` (global, >= t/4 entries), then the CTA radix select and a block-order sort.  For rows the
// split lists cannot settle (adversarial score orders): about a millisecond per 1M-token row.
struct ExactSmem {
  static constexpr int Q = 4 * 128 * 4;  // queries as fp32
  static constexpr int W = 16;
  static constexpr int HIST = 2048 * 4;
  static constexpr int RED = 48 * 8;
  static constexpr int WSUM = 32 * 4;
  static constexpr int SEL3 = 16;
  static constexpr int BLK = 512 * 4;
  static constexpr int SC = 512 * 4;
  static constexpr int TOTAL = Q + W + HIST + RED + WSUM + SEL3 + BLK + SC + 16;
};

__device__ __forceinline__ void exact_row_body(const ScoreArgs& a, const int row, u64* keys, uint8_t* smem) {
  float* sq = reinterpret_cast<float*>(smem);
  float* sw = sq + 4 * 128;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + ExactSmem::Q + ExactSmem::W);
  u64* red = reinterpret_cast<u64*>(smem + ExactSmem::Q + ExactSmem::W + ExactSmem::HIST);
  uint32_t* wsum = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(red) + ExactSmem::RED);
  uint32_t* sel3 = wsum + 32;
  uint32_t* sblk = sel3 + 4;
  float* ssc = reinterpret_cast<float*>(sblk + 512);
  int* cnt = reinterpret_cast<int*>(ssc + 512);
  const int tid = threadIdx.x;
  const int seq = a.q_seq[row], pos = a.q_pos[row];
  const int lim = pos / 4;
  const int need = min(a.topk, lim);
  for (int i = tid; i < 4 * 128; i += DM_THREADS)
    sq[i] = __bfloat162float(a.idx_q[(long long)row * 4 * 128 + i]);
  if (tid < 4) sw[tid] = __bfloat162float(a.idx_w[(long long)row * 4 + tid]);
  if (tid == 0) *cnt = 0;
  __syncthreads();
  const int32_t* pt = a.page_table + (long long)seq * a.max_pages;
  for (int b = tid; b < lim; b += DM_THREADS) {
    const int page = pt[b >> 4];
    float sc = 0.f;
    if (page >= 0 && page < a.num_pages) {
      const uint4* k4 = reinterpret_cast<const uint4*>(a.kcomp + ((long long)page * 16 + (b & 15)) * 128);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c = 0; c < 16; ++c) {
        const uint4 v = k4[c];
        const bf16* kh = reinterpret_cast<const bf16*>(&v);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float kd = __bfloat162float(kh[e]);
#pragma unroll
          for (int h = 0; h < 4; ++h) acc[h] = fmaf(sq[h * 128 + c * 8 + e], kd, acc[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < 4; ++h) sc = fmaf(sw[h], fmaxf(acc[h], 0.f), sc);
    } else {
      flag_error(a.err, QSA_DEVERR_PAGE);
    }
    keys[b] = make_key(sc, (uint32_t)b);
  }
  __syncthreads();
  const u64 kth = need > 0 ? cta_kth_largest(keys, lim, need, hist, red, wsum, sel3) : ~0ull;
  for (int b = tid; b < lim; b += DM_THREADS) {
    const u64 k = keys[b];
    if (need > 0 && k >= kth) {
      const int i = atomicAdd(cnt, 1);
      if (i < 512) {
        sblk[i] = (uint32_t)b;
        ssc[i] = key_score(k);
      }
    }
  }
  __syncthreads();
  if (tid < 32) {
    const int n = min(*cnt, need);
    if (n > 0) warp_sort_blocks(sblk, ssc, n);
    __syncwarp();
    write_selection(row, n, lim, sblk, ssc, a.sel, a.n_sel, a.sel_scores, a.sel_stride);
  }
  __syncthreads();
}

// ------------------------------------------------------------------ the fused decode step
// One cooperative launch, one CTA of 512 threads per SM, for a decode-sized batch:
//   compress   the step's new blocks (one 4-key group per CTA, first CTAs);
//   score      16 warps per CTA stream the compressed keys as dec_score_kernel does (warps whose
//              pages hold a block compressed in this launch wait for it first);
//   merge      CTA r selects row r exactly (dec_merge_body) once every CTA of its 4-row tile has
//              posted its lists, or, for a row the lists cannot settle, by the exact path;
//   attend     CTA i runs split i % S of row i / S once that row is selected (the swap-AB kernel
//              body; the last split of a row merges the partials);
// with no grid-wide barrier: each CTA waits (bounded, ~1 s) only on the counters or flags of the
// work it needs, in workspace words that are zero before the first call and that the last CTA to
// leave sets back to zero.
constexpr int FS_WARPS = 16;
constexpr int FS_THREADS = FS_WARPS * 32;
static_assert(FS_THREADS == DM_THREADS, "the merge body runs on the whole fused CTA");

struct StepSync {
  int* comp_done;   // [1] compressed groups
  int* tile_done;   // [T] score CTAs finished per 4-row tile
  int* merged;      // [num_q] row selected
  int* exit_count;  // [1] CTAs that left
};

struct StepArgs {
  ScoreArgs sa;
  AttnArgs aa;
  DecWs ws;
  int W, chunk, nl, lk, T;
  const bf16* idx_k_new;
  const int32_t* new_seq;
  const int32_t* new_pos;
  int n_groups;
  bf16* kcomp_w;
  u64* exact_keys;
  long long exact_ld;
  StepSync sync;
};

__device__ __forceinline__ void inval_mbar(uint8_t* p) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];\n" ::"r"(smem_addr(p)) : "memory");
}

// The merge's mbarrier, inside the MergeSmem layout.
constexpr int kMergeBarOff = MergeSmem::KEYS + MergeSmem::BOUNDS + MergeSmem::HIST + MergeSmem::CAND +
                             MergeSmem::LISTS + 448;
constexpr int kMergeKernelSmem = MergeSmem::TOTAL > ExactSmem::TOTAL ? MergeSmem::TOTAL : ExactSmem::TOTAL;

// One CTA per query row: the split-list merge, and for a row the lists cannot settle, the exact
// selection over every candidate in the same CTA (exact_keys: the row's candidate keys,
// exact_ld per row), so that no further launch has to look at the redo flags.
__global__ void __launch_bounds__(DM_THREADS) dec_merge_kernel(ScoreArgs a, DecWs ws, int nl, int lk,
                                                              u64* exact_keys, long long exact_ld) {
  extern __shared__ __align__(128) uint8_t smem[];
  chain_wait();
  chain_release();
  const int row = blockIdx.x;
  dec_merge_body(a, ws, nl, lk, row, smem);
  __syncthreads();
  const bool redo = *reinterpret_cast<volatile int32_t*>(&ws.redo[row]) != 0;
  if (!redo) return;  // uniform over the CTA
  if (threadIdx.x == 0) inval_mbar(smem + kMergeBarOff);  // its bytes are reused below
  __syncthreads();
  exact_row_body(a, row, exact_keys + (long long)row * exact_ld, smem);
}

// Bounded wait (thread 0) for *w >= target; then acquire and make generic-proxy writes visible to
// the async proxy.  Gives up after the wait limit with QSA_DEVERR_TIMEOUT.
__device__ __forceinline__ void wait_geq(const int* w, int target, int32_t* err) {
  const volatile int* v = w;
  if (*v < target) {
    const long long t0 = clock64();
    while (*v < target) {
      if (clock64() - t0 > kWaitLimitCycles) {
        flag_error(err, QSA_DEVERR_TIMEOUT);
        break;
      }
    }
  }
  __threadfence();
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}

template <int D, int HKV, int SLC>
__global__ void __launch_bounds__(FS_THREADS, 1)
    decode_step_kernel(StepArgs p, const __grid_constant__ CUtensorMap tmK) {
  extern __shared__ __align__(128) uint8_t smem[];
  using AC = SwCfg<D, HKV, SLC>;
  const int tid = threadIdx.x;
  const ScoreArgs& a = p.sa;

  // ---- compress: group g (4 raw keys of one block) by 16 threads of CTA g % gridDim.x
  int mine = 0;
  for (int g = blockIdx.x; g < p.n_groups; g += gridDim.x) {
    ++mine;
    if (tid < 16) {
      const long long r0 = (long long)g * 4;
      const int seq = p.new_seq[r0], pos0 = p.new_pos[r0];
      bool ok = pos0 >= 0 && pos0 % 4 == 0 && seq >= 0 && seq < a.batch && pos0 / 64 < a.max_pages;
#pragma unroll
      for (int i = 1; i < 4; ++i) ok = ok && p.new_seq[r0 + i] == seq && p.new_pos[r0 + i] == pos0 + i;
      const int page = ok ? a.page_table[(long long)seq * a.max_pages + pos0 / 64] : -1;
      if (ok && page >= 0 && page < a.num_pages) {
        double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = reinterpret_cast<const uint4*>(p.idx_k_new + (r0 + i) * 128)[tid];
          const bf16* h = reinterpret_cast<const bf16*>(&v);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += (double)__bfloat162float(h[e]);
        }
        uint4 o;
        bf16* oh = reinterpret_cast<bf16*>(&o);
#pragma unroll
        for (int e = 0; e < 8; ++e) oh[e] = __double2bfloat16(acc[e] * 0.25);
        reinterpret_cast<uint4*>(p.kcomp_w + ((long long)page * 16 + (pos0 / 4) % 16) * 128)[tid] = o;
      } else if (tid == 0) {
        flag_error(a.err, ok ? QSA_DEVERR_PAGE : QSA_DEVERR_GROUP);
      }
    }
  }
  if (mine) {
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      asm volatile("fence.proxy.async.global;\n" ::: "memory");
      atomicAdd(p.sync.comp_done, mine);
    }
  }

  // ---- score: virtual CTAs of FS_WARPS warps, one per CTA while they last
  NewBlockWait nbw;
  nbw.ctr = p.sync.comp_done;
  nbw.target = p.n_groups;
  nbw.new_seq = p.new_seq;
  nbw.new_pos = p.new_pos;
  nbw.n_groups = p.n_groups;
  // two virtual CTAs of DS_WARPS warps per block, as the standalone kernel runs two CTAs per SM:
  // a half that finishes its chunk folds its lists while the other half still streams
  const int per_tile = p.W / DS_WARPS;
  const int half = tid / DS_THREADS, htid = tid % DS_THREADS;
  uint8_t* hsmem = smem + half * DecSmem::TOTAL;
  for (int vb0 = 2 * blockIdx.x; vb0 < p.T * per_tile; vb0 += 2 * gridDim.x) {
    const int vb = vb0 + half;
    if (vb < p.T * per_tile) {
      dec_score_body<DS_WARPS>(a, &tmK, p.ws, p.W, p.chunk, p.nl, vb, hsmem, nbw, htid, 1 + half);
      asm volatile("bar.sync %0, %1;\n" ::"r"(1 + half), "n"(DS_THREADS) : "memory");
      if (htid < DS_WARPS * DS_NST) {  // the body's mbarriers, before the memory is reused
        uint8_t* al = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(hsmem) + 1023) & ~uintptr_t(1023));
        inval_mbar(al + DecSmem::STAGES + DecSmem::BUF + DecSmem::MLIST + DecSmem::MBOUND + DecSmem::PID +
                   htid * 8);
      }
      if (htid == 0) {
        __threadfence();
        atomicAdd(&p.sync.tile_done[vb / per_tile], 1);
      }
    }
    __syncthreads();
  }

  // ---- merge: row r by CTA r % gridDim.x, once its tile's lists are all posted
  for (int row = blockIdx.x; row < a.num_q; row += gridDim.x) {
    if (tid == 0) wait_geq(&p.sync.tile_done[row / 4], per_tile, a.err);
    __syncthreads();
    dec_merge_body(a, p.ws, p.nl, p.lk, row, smem);
    __syncthreads();
    if (tid == 0) inval_mbar(smem + kMergeBarOff);
    const bool redo = *reinterpret_cast<volatile int32_t*>(&p.ws.redo[row]) != 0;
    __syncthreads();
    if (redo) exact_row_body(a, row, p.exact_keys + (long long)row * p.exact_ld, smem);
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      atomicExch(&p.sync.merged[row], 1);
    }
  }

  // ---- attend: split i % S of row i / S, once the row is selected
  const int S = p.aa.splits;
  for (int it = blockIdx.x; it < a.num_q * S; it += gridDim.x) {
    const int row = it / S, split = it % S;
    if (tid == 0) wait_geq(&p.sync.merged[row], 1, a.err);
    __syncthreads();
    if (tid < AC::THREADS) sparse_attn_sw_body<D, HKV, SLC>(p.aa, row, split, smem);
    __syncthreads();
    if (tid < 2 * AC::NST + 1) inval_mbar(smem + AC::BAR_OFF + tid * 8);
    __syncthreads();
  }

  // ---- the last CTA out sets the sync words back to zero for the next launch
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(p.sync.exit_count, 1) == (int)gridDim.x - 1) {
      *p.sync.comp_done = 0;
      for (int t = 0; t < p.T; ++t) p.sync.tile_done[t] = 0;
      for (int r = 0; r < a.num_q; ++r) p.sync.merged[r] = 0;
      __threadfence();
      *p.sync.exit_count = 0;
    }
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

// The three-call form's workspace: the lists, bounds and redo flags, then every row's candidate
// keys for the merge kernel's exact path ((max_pos/4 + 1) keys per row).
long long dec_exact_ld(const Geometry& g) { return (long long)g.max_pos / 4 + 1; }

size_t dec_exact_offset(const Geometry& g, const DecPlan& p) {
  return stream_region(g) + r256((size_t)p.T * 4 * p.nl * p.lk * 8) + r256((size_t)p.T * 4 * pad2(p.nl) * 8) +
         r256((size_t)g.num_q * 4);
}

size_t score_dec_workspace_bytes(const Geometry& g) {
  DecPlan p;
  if (!dec_plan(g, &p)) return 0;
  return dec_exact_offset(g, p) + r256((size_t)g.num_q * dec_exact_ld(g) * 8);
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
  e = set_smem_once(dec_merge_kernel, kMergeKernelSmem);
  if (e != cudaSuccess) return e;
  const int warps = p.T * p.W;
  e = launch_chained(dec_score_kernel, dim3(warps / DS_WARPS), dim3(DS_THREADS), DecSmem::TOTAL, s, a, tmK, w, p.W,
                     p.chunk, p.nl);
  if (e != cudaSuccess) return e;
  u64* exact_keys = reinterpret_cast<u64*>(static_cast<uint8_t*>(ws) + dec_exact_offset(g, p));
  return launch_chained(dec_merge_kernel, dim3(g.num_q), dim3(DM_THREADS), kMergeKernelSmem, s, a, w, p.nl, p.lk,
                        exact_keys, dec_exact_ld(g));
}

// ------------------------------------------------------------------ fused decode step (host)
namespace {

struct StepLayout {
  DecPlan plan;
  int splits, grid;
  size_t dec, attn, keys, sync, total;
  long long exact_ld;
};

int step_grid() { return num_sms(); }  // one CTA of FS_THREADS per SM

bool step_layout(const Geometry& g, int num_splits, StepLayout* L) {
  L->grid = step_grid();
  if (!dec_plan_nw(g, DS_WARPS, (long long)L->grid * FS_WARPS, &L->plan)) return false;
  L->splits = resolve_sparse_splits(g, num_splits);
  const DecPlan& p = L->plan;
  L->dec = stream_region(g) + r256((size_t)p.T * 4 * p.nl * p.lk * 8) + r256((size_t)p.T * 4 * pad2(p.nl) * 8) +
           r256((size_t)g.num_q * 4);
  L->attn = r256(sparse_decode_workspace_bytes(g, L->splits));
  L->exact_ld = (long long)g.max_pos / 4 + 1;
  L->keys = r256((size_t)g.num_q * L->exact_ld * 8);
  L->sync = r256((size_t)(2 + p.T + 2 * g.num_q) * 4);
  L->total = L->dec + L->attn + L->keys + L->sync;
  return true;
}

template <int D, int HKV>
cudaError_t launch_step_kernel(const StepArgs& p, const CUtensorMap& tmK, int grid, cudaStream_t s) {
  constexpr int SLC = kSwSlices<HKV>;
  using AC = SwCfg<D, HKV, SLC>;
  int smem = 2 * DecSmem::TOTAL;
  smem = smem > MergeSmem::TOTAL ? smem : MergeSmem::TOTAL;
  smem = smem > ExactSmem::TOTAL ? smem : ExactSmem::TOTAL;
  smem = smem > AC::TOTAL ? smem : AC::TOTAL;
  cudaError_t e = set_smem_once(decode_step_kernel<D, HKV, SLC>, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(FS_THREADS);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the waits between them end
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_step_kernel<D, HKV, SLC>, p, tmK);
}

}  // namespace

bool decode_step_supported(const Geometry& g) {
  StepLayout L;
  return g.Di == 128 && g.G <= 8 && g.topk <= 512 && g.num_q <= 256 && step_layout(g, 0, &L);
}

size_t decode_step_workspace_bytes(const Geometry& g, int num_splits) {
  StepLayout L;
  if (!step_layout(g, num_splits, &L)) return 0;
  return L.total;
}

cudaError_t launch_decode_step(const Geometry& g, const void* idx_k_new, const int32_t* new_seq,
                               const int32_t* new_pos, int n_new, void* kcomp, const void* idx_q,
                               const void* idx_w, const void* q, const void* k_pool,
                               const void* v_pool, int32_t* sel, int32_t* n_sel, float* sel_scores,
                               void* out, float* lse, int num_splits, void* ws, cudaStream_t s) {
  auto enc = tmap_encode_fn();
  StepLayout L;
  if (!enc || !step_layout(g, num_splits, &L)) return cudaErrorNotSupported;
  uint8_t* base = static_cast<uint8_t*>(ws);
  StepArgs p;
  p.sa = make_args(g, idx_q, idx_w, kcomp, sel, n_sel, sel_scores);
  p.ws = carve_dec(g, L.plan, base);
  p.W = L.plan.W;
  p.chunk = L.plan.chunk;
  p.nl = L.plan.nl;
  p.lk = L.plan.lk;
  p.T = L.plan.T;
  p.idx_k_new = static_cast<const bf16*>(idx_k_new);
  p.new_seq = new_seq;
  p.new_pos = new_pos;
  p.n_groups = n_new / 4;
  p.kcomp_w = static_cast<bf16*>(kcomp);
  p.exact_keys = reinterpret_cast<u64*>(base + L.dec + L.attn);
  p.exact_ld = L.exact_ld;
  int* sync = reinterpret_cast<int*>(base + L.dec + L.attn + L.keys);
  p.sync.comp_done = sync;
  p.sync.exit_count = sync + 1;
  p.sync.tile_done = sync + 2;
  p.sync.merged = sync + 2 + L.plan.T;
  uint32_t* departures = reinterpret_cast<uint32_t*>(sync + 2 + L.plan.T + g.num_q);
  AttnArgs& aa = p.aa;
  aa.q = static_cast<const bf16*>(q);
  aa.k_pool = static_cast<const bf16*>(k_pool);
  aa.v_pool = static_cast<const bf16*>(v_pool);
  aa.sel = sel;
  aa.n_sel = n_sel;
  aa.sel_stride = g.topk + 1;
  aa.q_seq = g.q_seq;
  aa.q_pos = g.q_pos;
  aa.page_table = g.page_table;
  aa.num_q = g.num_q;
  aa.batch = g.batch;
  aa.max_pages = g.max_pages;
  aa.num_pages = g.num_pages;
  aa.Hq = g.Hq;
  aa.G = g.G;
  aa.scale_log2 = g.scale_log2;
  aa.out = static_cast<bf16*>(out);
  aa.lse = lse;
  aa.splits = L.splits;
  aa.err = g.err;
  aa.part_o = nullptr;
  aa.part_lse = nullptr;
  aa.arrivals = nullptr;
  aa.coop = (long long)g.num_q * L.splits <= L.grid;  // one split per CTA: all resident at once
  aa.departures = departures;
  if (L.splits > 1) {
    const size_t n = (size_t)g.num_q * L.splits * g.Hq;
    uint8_t* ab = base + L.dec;
    aa.part_o = reinterpret_cast<float*>(ab);
    aa.part_lse = reinterpret_cast<float*>(ab + ((n * g.D * 4 + 255) / 256) * 256);
    aa.arrivals = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(aa.part_lse) + ((n * 4 + 255) / 256) * 256);
  }
  CUtensorMap tmK;
  {
    cuuint64_t dims[2] = {128, (cuuint64_t)g.num_pages * 16};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, 16};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kcomp, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
#define QSA_STEP_CASE(DD, HH) \
  if (g.D == DD && g.Hkv == HH) return launch_step_kernel<DD, HH>(p, tmK, L.grid, s);
  QSA_STEP_CASE(128, 4)
  QSA_STEP_CASE(128, 8)
  QSA_STEP_CASE(128, 2)
  QSA_STEP_CASE(128, 1)
  QSA_STEP_CASE(64, 4)
  QSA_STEP_CASE(64, 8)
  QSA_STEP_CASE(64, 2)
  QSA_STEP_CASE(64, 1)
#undef QSA_STEP_CASE
  return cudaErrorNotSupported;
}

}  // namespace qsa
