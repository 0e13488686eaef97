// The comparison baseline, prefill form, on the 5th-generation tensor cores: dense causal paged
// grouped-query attention over every position <= t with tcgen05 MMAs into tensor memory.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "Three speed claims,
// three different experiments": the QSA module's speedups are quoted against paged grouped-query
// attention.  This is that baseline on the same paged pools (head_dim 128).
//
// CTA = two query tiles (A and B) of M = 128 rows each, sharing every K/V tile: a tile's 64 KB
// of keys and values feeds 2 x 8.4 MFLOP.  A query tile is TQ = 128 / G consecutive tokens x the G
// query heads of one KV head (row = token * G + head).  Warp-specialised:
//   warp 0      TMA producer: the two query tiles once (64 KB), then K and V tiles of 128
//               positions (two 64-token pages) of the KV head into a 2-stage ring (64 KB each);
//   warp 1      owns the tensor memory (per query tile: S/P 128 columns, O 128 columns) and one
//               lane issues, per query tile q and K/V tile j: O_q += P_q(j) V_j (P read from
//               tensor memory, V as an MN-major operand), then S_q(j+1) = Q_q K_{j+1}^T into the
//               same columns that held S_q(j) and P_q(j) (MMAs of one thread run in issue order);
//               the two query tiles alternate, so that one tile's softmax overlaps the other's MMAs;
//   warps 2-5 / 6-9  softmax of query tile A / B, one row per thread: two reads of S_q(j) (the
//               row maximum, then the exponentials), mask positions after t, keep the row's
//               reference maximum in base 2 (raised, with O and the running sum rescaled, only when
//               a tile's maximum exceeds it by more than 8: lazy rescaling), and write
//               P = 2^(scale * s - m) as bf16 pairs over the tile's own S columns; at the end
//               O / l and the log-sum-exp.  A tile that every row of the warp sees whole (all but
//               the last few of a segment) takes a path with no mask code and a three-input
//               maximum: the softmax's instruction stream, not a pipe, set the pace.
// Rows of a CTA that belong to different sequences are handled one sequence (segment) at a time.
// Cache slots after a segment's last position may be unwritten: their V rows are zeroed in the
// last tile before the MMA reads them, so a masked probability (0) never meets a non-finite value.
#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"
#include "tc_common.cuh"

namespace qsa {
namespace {

constexpr int DT_ROWS = 128;  // MMA M (one query tile)
constexpr int DT_NQ = 2;      // query tiles per CTA
constexpr int DT_POS = 128;   // positions per K/V tile: N of S, K of P V
constexpr int DT_NST = 2;     // K/V stages
constexpr int DT_SMW = 4;     // softmax warps per query tile
constexpr int DT_THREADS = (2 + DT_NQ * DT_SMW) * 32;
constexpr int DT_HALF = DT_ROWS * 128;         // one 64-column (128-byte) half of a 128-row tile
constexpr int DT_Q_BYTES = 2 * DT_HALF;        // one query tile, K-major: [k-half][row][128 B]
constexpr int DT_KV_BYTES = 2 * DT_HALF;       // K tile [k-half][position][128 B];
                                               // V tile [page][dim-half][64 positions][128 B]
constexpr int DT_STAGE = 2 * DT_KV_BYTES;      // K + V
constexpr float DT_RESCALE = 8.f;              // lazy rescaling threshold (base-2 exponent)
constexpr uint32_t kIdescS = idesc_bf16(DT_ROWS, DT_POS, false);
constexpr uint32_t kIdescPV = idesc_bf16(DT_ROWS, 128, true);

struct DtMisc {
  uint64_t qload, kv_full[DT_NST], kv_empty[DT_NST], s_full[DT_NQ], p_full[DT_NQ], o_done[DT_NQ];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int issued, consumed;  // K/V tiles issued by the producer / waited for by the MMA issuer
  int seg, tmax, ntile;
  uint32_t done[8];   // tokens already handled (bit per token)
  uint32_t inseg[8];  // tokens of the current segment
};
constexpr int DT_SMEM = DT_NQ * DT_Q_BYTES + DT_NST * DT_STAGE + (int)((sizeof(DtMisc) + 127) / 128 * 128);
static_assert(DT_SMEM <= 232448, "shared memory budget");

struct DtArgs {
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int num_q, batch, max_pages, num_pages, Hq, Hkv, G, TQ;
  float scale_log2;
  bf16* out;
  float* lse;
  int32_t* err;
};

// 2^x on the special-function unit (flush-to-zero, about 2 ulp): plenty for bf16 probabilities.
// Largest of three (Blackwell's three-input max): half the instructions of a max tree.
__device__ __forceinline__ float fmax3(float x, float y, float z) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(x), "f"(y), "f"(z));
  return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool dt_bit(const uint32_t* b, int i) { return (b[i >> 5] >> (i & 31)) & 1u; }

__global__ void __launch_bounds__(DT_THREADS, 1)
    dense_tc_kernel(DtArgs a, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + DT_NQ * DT_Q_BYTES;
  DtMisc* m = reinterpret_cast<DtMisc*>(sKV + DT_NST * DT_STAGE);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int TQ = a.TQ, G = a.G;
  const int NT = DT_NQ * TQ;  // tokens of the CTA
  const int tok0 = blockIdx.x * NT;
  const int g = blockIdx.y;

  if (smem_addr(smem) & 1023) {  // operand tiles need 1024-byte alignment
    if (tid == 0) flag_error(a.err, QSA_DEVERR_INTERNAL);
    return;
  }
  if (tid == 0) {
    mbar_init(&m->qload, 1);
    for (int s = 0; s < DT_NST; ++s) {
      mbar_init(&m->kv_full[s], 1);
      mbar_init(&m->kv_empty[s], 1);
    }
    for (int q = 0; q < DT_NQ; ++q) {
      mbar_init(&m->s_full[q], 1);
      mbar_init(&m->p_full[q], DT_SMW);
      mbar_init(&m->o_done[q], 1);
    }
    mbar_init(&m->mma_done, 1);
    m->abort_flag = 0;
    m->issued = 0;
    m->consumed = 0;
    for (int i = 0; i < 8; ++i) m->done[i] = 0;
    // tokens that fail validation are done from the start (their rows are never written)
    for (int i = 0; i < NT; ++i) {
      const int r = tok0 + i;
      bool bad = r >= a.num_q;
      if (!bad) {
        const int s = a.q_seq[r], t = a.q_pos[r];
        if (s < 0 || s >= a.batch || t < 0 || t / 64 >= a.max_pages) {
          flag_error(a.err, (s < 0 || s >= a.batch) ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);
          bad = true;
        }
      }
      if (bad) m->done[i >> 5] |= 1u << (i & 31);
    }
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
    mbar_arrive_expect_tx(&m->qload, DT_NQ * DT_Q_BYTES);
    for (int q = 0; q < DT_NQ; ++q)
      for (int kh = 0; kh < 2; ++kh)
        tma3d(smem_addr(sQ + q * DT_Q_BYTES + kh * DT_HALF), &tmQ, kh * 64, g * G, tok0 + q * TQ, &m->qload);
  }

  // softmax thread: query tile qt, row (TMEM lane quarter warp % 4)
  const int qt = warp >= 2 ? (warp - 2) / DT_SMW : 0;
  const int row = 32 * (warp & 3) + lane;
  const int tok = qt * TQ + row / G, head = row % G;
  const uint32_t tS = tbase + qt * 256, tO = tS + 128;  // this query tile's S/P and O columns

  int gbase = 0;  // tiles of earlier segments (every role counts the same tiles)
  for (;;) {
    __syncthreads();
    if (tid == 0) {  // next segment: the sequence of the first token not yet done
      int seg = -1, tmax = -1;
      for (int i = 0; i < 8; ++i) m->inseg[i] = 0;
      for (int i = 0; i < NT; ++i) {
        if (dt_bit(m->done, i)) continue;
        const int s = a.q_seq[tok0 + i];
        if (seg < 0) seg = s;
        if (s == seg) {
          m->inseg[i >> 5] |= 1u << (i & 31);
          tmax = max(tmax, a.q_pos[tok0 + i]);
        }
      }
      m->seg = seg;
      m->tmax = tmax;
      m->ntile = seg < 0 ? 0 : tmax / DT_POS + 1;
    }
    __syncthreads();
    const int seg = m->seg;
    if (seg < 0 || m->abort_flag) break;
    const int ntile = m->ntile, seg_tmax = m->tmax;

    if (warp == 0) {
      // ---------------------------------------------------------------- TMA producer
      if (lane == 0) {
        const int32_t* pt = a.page_table + (long long)seg * a.max_pages;
        for (int j = 0; j < ntile; ++j) {
          const int gj = gbase + j, s = gj % DT_NST;
          if (gj >= DT_NST && !mbar_wait(&m->kv_empty[s], ((gj / DT_NST) & 1) ^ 1, a.err)) {
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
          uint8_t* st = sKV + s * DT_STAGE;
          mbar_arrive_expect_tx(&m->kv_full[s], DT_STAGE);
          for (int pg = 0; pg < 2; ++pg)
            for (int hh = 0; hh < 2; ++hh) {
              // K: [k-half hh][positions pg*64..][128 B];  V: [page pg][dim-half hh][64][128 B]
              tma3d(smem_addr(st + hh * DT_HALF + pg * (DT_HALF / 2)), &tmK, hh * 64, g, pid[pg] * 64,
                    &m->kv_full[s]);
              tma3d(smem_addr(st + DT_KV_BYTES + pg * DT_HALF + hh * (DT_HALF / 2)), &tmV, hh * 64, g,
                    pid[pg] * 64, &m->kv_full[s]);
            }
          m->issued = gj + 1;
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        bool ok = gbase > 0 || mbar_wait(&m->qload, 0, a.err);
        auto s_mma = [&](int q, int j) {  // S_q(j) = Q_q K_j^T
          const uint32_t qa = smem_addr(sQ + q * DT_Q_BYTES);
          const uint32_t kb = smem_addr(sKV + ((gbase + j) % DT_NST) * DT_STAGE);
#pragma unroll
          for (int ks = 0; ks < 128 / 16; ++ks) {
            const uint64_t ad = sw128_desc(qa + (ks >> 2) * DT_HALF + (ks & 3) * 32);
            const uint64_t bd = sw128_desc(kb + (ks >> 2) * DT_HALF + (ks & 3) * 32);
            umma_bf16(tbase + q * 256, ad, bd, kIdescS, ks > 0 ? 1u : 0u);
          }
          umma_commit(&m->s_full[q]);
        };
        auto load_ready = [&](int j) -> bool {
          const int gj = gbase + j;
          if (!mbar_wait(&m->kv_full[gj % DT_NST], (gj / DT_NST) & 1, a.err)) return false;
          m->consumed = gj + 1;
          tc_fence_after();
          return true;
        };
        if (ok && load_ready(0))
          for (int q = 0; q < DT_NQ; ++q) s_mma(q, 0);
        else
          ok = false;
        for (int j = 0; ok && j < ntile; ++j) {
          const int gj = gbase + j;
          const uint32_t vb = smem_addr(sKV + (gj % DT_NST) * DT_STAGE + DT_KV_BYTES);
          for (int q = 0; ok && q < DT_NQ; ++q) {
            if (!mbar_wait(&m->p_full[q], gj & 1, a.err)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < DT_POS / 16; ++ks) {  // O_q (+)= P_q(j) V_j
              const uint64_t bd = sw128_desc_mn(vb + (ks >> 2) * DT_HALF + (ks & 3) * 2048, DT_HALF / 2);
              umma_bf16_ts(tbase + q * 256 + 128, tbase + q * 256 + ks * 8, bd, kIdescPV,
                           (j > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit(&m->o_done[q]);
            if (j + 1 < ntile) {
              if (q == 0 && !load_ready(j + 1)) { ok = false; break; }
              s_mma(q, j + 1);  // overwrites S_q(j) / P_q(j): after the PV above, in issue order
            }
          }
          if (ok) umma_commit(&m->kv_empty[gj % DT_NST]);
        }
        if (!ok) m->abort_flag = 1;
      }
    } else {
      // ---------------------------------------------------------------- softmax
      const bool act = dt_bit(m->inseg, tok);
      const int t = act ? a.q_pos[tok0 + tok] : -1;
      const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;  // TMEM lane base of this warp
      float m_ref = -INFINITY, l_sum = 0.f;
      // A warp that gives up waiting (error flagged) goes on without its waits and tensor-memory
      // accesses, with `dead` warp-uniform, so that the collective accesses stay uniform.
      bool dead = false;
      auto waitw = [&](uint64_t* bar, uint32_t par) {
        if (dead) return;
        const bool okw = mbar_wait(bar, par, a.err);
        if (__any_sync(0xffffffffu, !okw)) {
          m->abort_flag = 1;
          dead = true;
        }
      };
      for (int j = 0; j < ntile; ++j) {
        const int gj = gbase + j, s = gj % DT_NST;
        const int P0 = j * DT_POS;
        // S_q(j) is complete, and with it every earlier MMA (P_q(j-1) has been read, O_q holds
        // tiles < j)
        waitw(&m->s_full[qt], gj & 1);
        const bool vis = P0 + DT_POS - 1 <= t;  // whole tile visible: no mask
        const bool allvis = __all_sync(0xffffffffu, vis);  // every row of the warp: no mask code
        // pass 1: the row maximum
        float mx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
        if (!dead && allvis) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < DT_POS / 16; ++c) {
            float x[16];
            tmem_ld16(tS + lb + c * 16, x);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) mx[e] = fmax3(mx[e], x[e], x[e + 8]);
          }
        } else if (!dead) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < DT_POS / 16; ++c) {
            float x[16];
            tmem_ld16(tS + lb + c * 16, x);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float y = (vis || P0 + c * 16 + e <= t) ? x[e] : -INFINITY;
              mx[e & 7] = fmaxf(mx[e & 7], y);
            }
          }
        }
        const float tmx = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * a.scale_log2;
        const float m_new = fmaxf(m_ref, tmx);
        const bool resc = m_ref != -INFINITY && m_new > m_ref + DT_RESCALE;
        if (__any_sync(0xffffffffu, resc) && !dead) {  // rescale O_q: no MMA writes it now
          const float f = resc ? exp2f(m_ref - m_new) : 1.f;
#pragma unroll
          for (int c = 0; c < 128 / 16; ++c) {
            float o[16];
            tmem_ld16(tO + lb + c * 16, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= f;
            tmem_st16(tO + lb + c * 16, o);
          }
          tmem_wait_st();
        }
        if (resc) {
          l_sum *= exp2f(m_ref - m_new);
          m_ref = m_new;
        }
        if (m_ref == -INFINITY) m_ref = m_new;  // first visible tile (stays -inf if none)
        // pass 2: P = 2^(scale * s - m_ref) as bf16 pairs over columns 0..63 of the tile's S
        // (chunk c of 32 positions lands on S columns already read); a row with nothing visible
        // yet has every s masked to -inf and gets p = 0
        const float nm = m_ref == -INFINITY ? -INFINITY : -m_ref;
        float rsv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) rsv[e] = 0.f;
        if (!dead && allvis) {
#pragma unroll
          for (int c = 0; c < DT_POS / 32; ++c) {
            float x[16], y[16];
            tmem_ld16(tS + lb + c * 32, x);
            tmem_ld16(tS + lb + c * 32 + 16, y);
            tmem_wait_ld();
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float a0 = e < 8 ? x[2 * e] : y[2 * e - 16];
              const float a1 = e < 8 ? x[2 * e + 1] : y[2 * e - 15];
              const float e0 = fast_exp2(fmaf(a0, a.scale_log2, nm));
              const float e1 = fast_exp2(fmaf(a1, a.scale_log2, nm));
              rsv[e & 7] += e0 + e1;
              w[e] = pack_bf16(e0, e1);
            }
            tmem_st16u(tS + lb + c * 16, w);
          }
          tmem_wait_st();
        } else if (!dead) {
#pragma unroll
          for (int c = 0; c < DT_POS / 32; ++c) {
            float x[16], y[16];
            tmem_ld16(tS + lb + c * 32, x);
            tmem_ld16(tS + lb + c * 32 + 16, y);
            tmem_wait_ld();
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int p0 = P0 + c * 32 + 2 * e;
              const float a0 = e < 8 ? x[2 * e] : y[2 * e - 16];
              const float a1 = e < 8 ? x[2 * e + 1] : y[2 * e - 15];
              const float e0 = fast_exp2(fmaf((vis || p0 <= t) ? a0 : -INFINITY, a.scale_log2, nm));
              const float e1 = fast_exp2(fmaf((vis || p0 + 1 <= t) ? a1 : -INFINITY, a.scale_log2, nm));
              rsv[e & 7] += e0 + e1;
              w[e] = pack_bf16(e0, e1);
            }
            tmem_st16u(tS + lb + c * 16, w);
          }
          tmem_wait_st();
        }
        l_sum += ((rsv[0] + rsv[1]) + (rsv[2] + rsv[3])) + ((rsv[4] + rsv[5]) + (rsv[6] + rsv[7]));
        if (P0 + DT_POS - 1 > seg_tmax && qt == 0) {
          // the segment's last tile: zero the V rows after its last position (query tile A's
          // softmax does it; B's PV is issued after A's)
          waitw(&m->kv_full[s], (gj / DT_NST) & 1);
          if (!dead && P0 + row > seg_tmax) {
            uint8_t* vr = sKV + s * DT_STAGE + DT_KV_BYTES + (row >> 6) * DT_HALF + (row & 63) * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              *reinterpret_cast<uint4*>(vr + c * 16) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(vr + DT_HALF / 2 + c * 16) = make_uint4(0, 0, 0, 0);
            }
          }
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // V for the MMA
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && !dead) mbar_arrive(&m->p_full[qt]);
      }
      if (ntile > 0) {
        const int gl = gbase + ntile - 1;
        waitw(&m->o_done[qt], gl & 1);
        if (!dead) {
          tc_fence_after();
          const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
          bf16* dst = act ? a.out + ((long long)(tok0 + tok) * a.Hq + g * G + head) * 128 : nullptr;
#pragma unroll
          for (int c = 0; c < 128 / 16; ++c) {
            float o[16];
            tmem_ld16(tO + lb + c * 16, o);
            tmem_wait_ld();
            if (act) {
              uint32_t w[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) w[e] = pack_bf16(o[2 * e] * inv, o[2 * e + 1] * inv);
              *reinterpret_cast<uint4*>(dst + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
              *reinterpret_cast<uint4*>(dst + c * 16 + 8) = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
          if (act && a.lse)
            a.lse[(long long)(tok0 + tok) * a.Hq + g * G + head] =
                l_sum > 0.f ? (m_ref + log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
          tc_fence_before();
        }
      }
    }
    __syncthreads();
    if (tid < 8) m->done[tid] |= m->inseg[tid];
    gbase += ntile;
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (m->abort_flag && warp == 0 && lane == 0) {  // let copies still in flight land first
    mbar_wait(&m->qload, 0, a.err);
    for (int gj = m->consumed; gj < m->issued; ++gj)
      mbar_wait(&m->kv_full[gj % DT_NST], (gj / DT_NST) & 1, a.err);
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

}  // namespace

bool dense_tc_supported(const Geometry& g) {
  return g.D == 128 && g.G >= 1 && g.G <= 128 && 128 % g.G == 0 && tmap_encode_fn() != nullptr;
}

cudaError_t launch_dense_tc(const Geometry& g, const void* q, const void* k_pool, const void* v_pool,
                            void* out, float* lse, cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  auto enc = tmap_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  DtArgs a;
  a.q_seq = g.q_seq;
  a.q_pos = g.q_pos;
  a.page_table = g.page_table;
  a.num_q = g.num_q;
  a.batch = g.batch;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.G = g.G;
  a.TQ = DT_ROWS / g.G;
  a.scale_log2 = g.scale_log2;
  a.out = static_cast<bf16*>(out);
  a.lse = lse;
  a.err = g.err;
  CUtensorMap tmQ, tmK, tmV;
  {
    cuuint64_t dims[3] = {128, (cuuint64_t)g.Hq, (cuuint64_t)g.num_q};
    cuuint64_t strides[2] = {256, (cuuint64_t)g.Hq * 256};
    cuuint32_t box[3] = {64, (cuuint32_t)g.G, (cuuint32_t)a.TQ};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  for (int kv = 0; kv < 2; ++kv) {
    cuuint64_t dims[3] = {128, (cuuint64_t)g.Hkv, (cuuint64_t)g.num_pages * 64};
    cuuint64_t strides[2] = {256, (cuuint64_t)g.Hkv * 256};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(kv ? &tmV : &tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv ? v_pool : k_pool),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = set_smem_once(dense_tc_kernel, DT_SMEM);
  if (e != cudaSuccess) return e;
  const int nt = DT_NQ * a.TQ;
  dense_tc_kernel<<<dim3((g.num_q + nt - 1) / nt, g.Hkv), DT_THREADS, DT_SMEM, s>>>(a, tmQ, tmK, tmV);
  return cudaGetLastError();
}

}  // namespace qsa
