// The indexer's dense-distillation signal: KL(teacher || indexer) per query row.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "The indexer is
// trained, not bolted on": before sparse training the indexer learned from the full-attention
// distribution, with token-level attention pooled into blocks as the teacher.  Readings (the
// article gives no formula): the teacher of query position t is the dense causal softmax
// attention of every core query head over positions 0..t, summed over the 4 tokens of each
// candidate block b < t/4 and over all query heads, renormalised over the candidates; the
// student is the softmax of the indexer's block scores s_b = sum_h w_h relu(q_h . k_b) over the
// same candidates; the loss is KL(teacher || student) in nats (0 for rows without candidates).
//
// One CTA owns TQ = min(16, 256 / Hq) query tokens of one sequence segment with all of their
// query heads: 256 MMA rows (token, head) ordered KV-head-major, so each 16-row m-tile reads a
// single KV head.  Two passes over the sequence's keys, both on mma.sync tiles of 32 positions
// (all KV heads of a page half, double-buffered by cp.async):
//   pass 1  online max / sum of every row's logits over positions 0..t -> each head's
//           log-sum-exp (optionally written out);
//   pass 2  the probabilities exp(z - lse) of candidate positions, summed within each block by
//           warp shuffles, over the heads of an m-tile by shuffles, over KV heads by shared-memory
//           atomics; the same tile's compressed keys give the student scores (a small MMA of the
//           token's 4 indexer heads); per (token, block) the masses m and scores s then update the
//           row's sums M = sum m, A = sum m log m, B = sum m s and the running log-sum-exp of s,
//           so that KL = A/M - log M - B/M + logsumexp(s) needs no stored distribution.
// The teacher distribution itself ([num_q, ld], m / M) is written only when asked for.
#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"

namespace qsa {
namespace {

constexpr int DL_THREADS = 256;
constexpr int DL_POS = 32;  // positions per tile = 8 micro-blocks
constexpr int DL_NST = 2;

struct DistillArgs {
  const bf16* q;
  const bf16* k_pool;
  const bf16* idx_q;
  const bf16* idx_w;
  const bf16* kcomp;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int num_q, batch, max_pages, num_pages, max_pos, Hq, Hkv, G, TQ;
  float scale_log2;
  float* kl;
  float* lse;
  float* teacher;
  long long ld;
  int32_t* err;
};

// Shared-memory layout (bytes), the same on host and device.
struct DlLayout {
  int q, iq, k, kc, f, total, kst, kcst;
  __host__ __device__ DlLayout(int D, int DI, int TQ, int Hq, int Hkv) {
    const int iq_rows = TQ * 4 > 16 ? TQ * 4 : 16;
    kst = DL_POS * Hkv * D * 2;
    kcst = 8 * DI * 2;
    q = 0;
    iq = q + TQ * Hq * D * 2;
    k = iq + iq_rows * DI * 2;
    kc = k + DL_NST * kst;
    f = kc + DL_NST * kcst;
    total = f + TQ * (8 + 8 + 4 + 1) * 4 + TQ * 2 * 4 + 16;
  }
};

template <int D, int DI>
__global__ void __launch_bounds__(DL_THREADS, 1) distill_kl_kernel(DistillArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int TQ = a.TQ, Hq = a.Hq, Hkv = a.Hkv, G = a.G;
  const DlLayout L(D, DI, TQ, Hq, Hkv);
  const int nmt = TQ * Hq / 16;       // m-tiles of (token, head) rows, <= 16
  const int rows_kv = TQ * G;         // rows per KV head, a multiple of 16
  const int iq_rows = TQ * 4 > 16 ? TQ * 4 : 16;
  const uint32_t base = smem_addr(smem);
  const uint32_t sQ = base + L.q, sIQ = base + L.iq, sK = base + L.k, sKC = base + L.kc;
  float* sMass = reinterpret_cast<float*>(smem + L.f);  // [TQ][8] teacher mass of the tile
  float* sStu = sMass + TQ * 8;                          // [TQ][8] student scores of the tile
  float* sW = sStu + TQ * 8;                             // [TQ][4] head weights
  float* sM = sW + TQ * 4;                               // [TQ] teacher total of the segment
  int* sT = reinterpret_cast<int*>(sM + TQ);             // [TQ] position, -1 outside the segment
  int* sSeq = sT + TQ;                                   // [TQ] sequence, -1 for invalid rows
  int* sMisc = sSeq + TQ;                                // segment, its largest position

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qr = lane >> 2, qc = lane & 3;
  const int row0 = blockIdx.x * TQ;

  if (tid < TQ) {
    const int r = row0 + tid;
    int s = -1;
    if (r < a.num_q) {
      const int sq = a.q_seq[r], t = a.q_pos[r];
      if (sq < 0 || sq >= a.batch) flag_error(a.err, QSA_DEVERR_SEQ);
      else if (t < 0 || t > a.max_pos || t / 64 >= a.max_pages) flag_error(a.err, QSA_DEVERR_POS);
      else s = sq;
      if (s < 0) a.kl[r] = __int_as_float(0x7fc00000);  // invalid row: NaN
    }
    sSeq[tid] = s;
#pragma unroll
    for (int h = 0; h < 4; ++h)
      sW[tid * 4 + h] = s >= 0 ? __bfloat162float(a.idx_w[(long long)r * 4 + h]) : 0.f;
  }
  for (int i = tid; i < TQ * 8; i += DL_THREADS) sMass[i] = 0.f;
  // the tile's queries ([row][D], row = kv * TQ*G + token * G + head-in-group) and indexer queries
  for (int i = tid; i < TQ * Hq * (D / 8); i += DL_THREADS) {
    const int R = i / (D / 8), c = i % (D / 8);
    const int kv = R / rows_kv, loc = R % rows_kv, tok = loc / G, hl = loc % G;
    const int r = row0 + tok;
    const bool valid = r < a.num_q;
    const bf16* src = valid ? a.q + ((long long)r * Hq + kv * G + hl) * D + c * 8 : a.q;
    cp_async16(sQ + R * (D * 2) + ((c ^ (R & 7)) << 4), src, valid);
  }
  for (int i = tid; i < iq_rows * (DI / 8); i += DL_THREADS) {
    const int R = i / (DI / 8), c = i % (DI / 8);
    const int tok = R / 4, r = row0 + tok;
    const bool valid = tok < TQ && r < a.num_q;
    const bf16* src = valid ? a.idx_q + ((long long)r * 4 + (R % 4)) * DI + c * 8 : a.idx_q;
    cp_async16(sIQ + swz<DI>(R, c), src, valid);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  unsigned done = 0;  // bit per token: handled, or invalid (the same in every thread)
  for (int i = 0; i < TQ; ++i)
    if (sSeq[i] < 0) done |= 1u << i;

  for (;;) {
    if (tid == 0) {
      int seg = -1, tmax = -1;
      for (int i = 0; i < TQ; ++i)
        if (!((done >> i) & 1u) && seg < 0) seg = sSeq[i];
      for (int i = 0; i < TQ; ++i)
        if (!((done >> i) & 1u) && sSeq[i] == seg && seg >= 0) tmax = max(tmax, a.q_pos[row0 + i]);
      sMisc[0] = seg;
      sMisc[1] = tmax;
    }
    __syncthreads();
    const int seg = sMisc[0], tmax = sMisc[1];
    if (seg < 0) break;
    if (tid < TQ) sT[tid] = (!((done >> tid) & 1u) && sSeq[tid] == seg) ? a.q_pos[row0 + tid] : -1;
    for (int i = 0; i < TQ; ++i)
      if (sSeq[i] == seg) done |= 1u << i;
    __syncthreads();

    const int32_t* ptab = a.page_table + (long long)seg * a.max_pages;
    const int nb_max = tmax / 4;  // candidate blocks of the segment's last row
    // 32 positions of all KV heads (one contiguous run of a page) and, in pass 2, the page's 8
    // compressed keys of the same positions
    auto load = [&](int it, int st, bool with_kc) {
      const int p0 = it * DL_POS;
      int page = ptab[p0 / 64];
      const bool ok = page >= 0 && page < a.num_pages;
      if (!ok) {
        if (tid == 0) flag_error(a.err, QSA_DEVERR_PAGE);
        page = 0;
      }
      const bf16* kb = a.k_pool + ((long long)page * 64 + (p0 % 64)) * Hkv * D;
      for (int i = tid; i < DL_POS * Hkv * (D / 8); i += DL_THREADS) {
        const int row = i / (D / 8), c = i % (D / 8), pl = row / Hkv;
        const bool valid = ok && p0 + pl <= tmax;
        cp_async16(sK + st * L.kst + row * (D * 2) + ((c ^ (pl & 7)) << 4),
                   valid ? kb + (long long)row * D + c * 8 : a.k_pool, valid);
      }
      if (with_kc) {
        const int b0 = p0 / 4;
        for (int i = tid; i < 8 * (DI / 8); i += DL_THREADS) {
          const int blk = i / (DI / 8), c = i % (DI / 8);
          const bool valid = ok && b0 + blk < nb_max;
          const bf16* src = a.kcomp + ((long long)page * 16 + ((b0 + blk) & 15)) * DI + c * 8;
          cp_async16(sKC + st * L.kcst + swz<DI>(blk, c), valid ? src : a.kcomp, valid);
        }
      }
    };

    // this thread's rows: m-tiles j = warp and warp + 8
    int kvj[2], toka[2], tokb[2], ta[2], tb[2];
    bool act[2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int j = warp + 8 * jj;
      act[jj] = j < nmt;
      const int Ra = 16 * j + qr, Rb = Ra + 8;
      kvj[jj] = act[jj] ? Ra / rows_kv : 0;
      toka[jj] = act[jj] ? (Ra % rows_kv) / G : 0;
      tokb[jj] = act[jj] ? (Rb % rows_kv) / G : 0;
      ta[jj] = act[jj] ? sT[toka[jj]] : -1;
      tb[jj] = act[jj] ? sT[tokb[jj]] : -1;
    }
    // S = Q K^T of m-tile j over the tile's 32 positions (4 n-tiles of 8)
    auto scores = [&](int j, int kv, int st, float (&sc)[4][4]) {
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
      const uint32_t kbase = sK + st * L.kst;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t af[4];
        const int R = 16 * j + (lane & 15);
        ldsm_x4(af, sQ + R * (D * 2) + (((ks * 2 + (lane >> 4)) ^ (R & 7)) << 4));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t kf[4];
          const int pl = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int c = ks * 2 + ((lane >> 3) & 1);
          ldsm_x4(kf, kbase + (pl * Hkv + kv) * (D * 2) + ((c ^ (pl & 7)) << 4));
          mma_bf16_16816(sc[2 * np], af, kf[0], kf[1]);
          mma_bf16_16816(sc[2 * np + 1], af, kf[2], kf[3]);
        }
      }
    };

    // ---------------------------------------------------------------- pass 1: log-sum-exp
    float mx[2][2], sm[2][2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[jj][h] = -INFINITY;
        sm[jj][h] = 0.f;
      }
    const int nt1 = tmax / DL_POS + 1;
    load(0, 0, false);
    cp_async_commit();
    for (int it = 0; it < nt1; ++it) {
      cp_async_wait<0>();
      __syncthreads();
      if (it + 1 < nt1) load(it + 1, (it + 1) & 1, false);
      cp_async_commit();
      const int p0 = it * DL_POS;
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        if (!act[jj] || !__any_sync(0xffffffffu, ta[jj] >= p0 || tb[jj] >= p0)) continue;
        float sc[4][4];
        scores(warp + 8 * jj, kvj[jj], it & 1, sc);
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = p0 + nt * 8 + 2 * qc + e;
            sc[nt][e] = p <= ta[jj] ? sc[nt][e] * a.scale_log2 : -INFINITY;
            sc[nt][2 + e] = p <= tb[jj] ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
            m0 = fmaxf(m0, sc[nt][e]);
            m1 = fmaxf(m1, sc[nt][2 + e]);
          }
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
        const float n0 = fmaxf(mx[jj][0], m0), n1 = fmaxf(mx[jj][1], m1);
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            s0 += n0 == -INFINITY ? 0.f : exp2f(sc[nt][e] - n0);
            s1 += n1 == -INFINITY ? 0.f : exp2f(sc[nt][2 + e] - n1);
          }
        sm[jj][0] = (n0 == -INFINITY ? 0.f : sm[jj][0] * exp2f(mx[jj][0] - n0)) + s0;
        sm[jj][1] = (n1 == -INFINITY ? 0.f : sm[jj][1] * exp2f(mx[jj][1] - n1)) + s1;
        mx[jj][0] = n0;
        mx[jj][1] = n1;
      }
    }
    cp_async_wait<0>();
    __syncthreads();
    float lse2[2][2];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float s = sm[jj][h];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        lse2[jj][h] = s > 0.f ? mx[jj][h] + log2f(s) : INFINITY;  // +inf: no probability
      }
      if (act[jj] && a.lse && qc == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int R = 16 * (warp + 8 * jj) + qr + 8 * h;
          const int loc = R % rows_kv, tok = loc / G;
          if (sT[tok] >= 0)
            a.lse[(long long)(row0 + tok) * Hq + kvj[jj] * G + loc % G] = lse2[jj][h] * 0.69314718055994531f;
        }
      }
    }

    // ---------------------------------------------------------------- pass 2: pooled KL
    const int gmin = G < 8 ? G : 8;
    double accM = 0.0, accA = 0.0, accB = 0.0, lmax = -INFINITY, lsum = 0.0;
    const int kl_tok = tid >> 3, kl_blk = tid & 7;  // KL bookkeeping: one thread per (token, block)
    const bool kl_thr = kl_tok < TQ;
    const int kl_t = kl_thr ? sT[kl_tok] : -1;
    const int nt2 = (4 * nb_max + DL_POS - 1) / DL_POS;
    if (nt2 > 0) {
      load(0, 0, true);
      cp_async_commit();
    }
    for (int it = 0; it < nt2; ++it) {
      cp_async_wait<0>();
      __syncthreads();
      if (it + 1 < nt2) load(it + 1, (it + 1) & 1, true);
      cp_async_commit();
      const int p0 = it * DL_POS, st = it & 1;
      // teacher: per-head probabilities of candidate positions, pooled per block
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int ca = 4 * (ta[jj] >> 2), cb = 4 * (tb[jj] >> 2);  // candidate positions < c
        if (!act[jj] || !__any_sync(0xffffffffu, ca > p0 || cb > p0)) continue;
        float sc[4][4];
        scores(warp + 8 * jj, kvj[jj], st, sc);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          float va = 0.f, vb = 0.f;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = p0 + nt * 8 + 2 * qc + e;
            va += p < ca ? exp2f(sc[nt][e] * a.scale_log2 - lse2[jj][0]) : 0.f;
            vb += p < cb ? exp2f(sc[nt][2 + e] * a.scale_log2 - lse2[jj][1]) : 0.f;
          }
          va += __shfl_xor_sync(0xffffffffu, va, 1);  // the block's 4 positions
          vb += __shfl_xor_sync(0xffffffffu, vb, 1);
          if (G >= 16) va += vb;                      // rows 8..15: the same token
          for (int o = 4; o < 4 * gmin; o <<= 1) {    // the heads of the token in this m-tile
            va += __shfl_xor_sync(0xffffffffu, va, o);
            vb += __shfl_xor_sync(0xffffffffu, vb, o);
          }
          if ((qc & 1) == 0 && qr % gmin == 0) {
            const int blk = 2 * nt + (qc >> 1);
            if (ta[jj] >= 0) atomicAdd(&sMass[toka[jj] * 8 + blk], va);
            if (G < 16 && tb[jj] >= 0) atomicAdd(&sMass[tokb[jj] * 8 + blk], vb);
          }
        }
      }
      // student: the indexer's scores of the tile's 8 blocks, (token, head) rows in m-tiles
      if (warp < iq_rows / 16) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < DI / 32; ++kk) {
          uint32_t bfr[4];
          ldsm_x4(bfr, sKC + st * L.kcst + swz<DI>(lane & 7, kk * 4 + (lane >> 3)));
#pragma unroll
          for (int s2 = 0; s2 < 2; ++s2) {
            uint32_t af[4];
            ldsm_x4(af, sIQ + swz<DI>(16 * warp + (lane & 15), (2 * kk + s2) * 2 + (lane >> 4)));
            mma_bf16_16816(acc, af, bfr[2 * s2], bfr[2 * s2 + 1]);
          }
        }
        const int Ra = 16 * warp + qr, Rb = Ra + 8;
        const float wa = Ra / 4 < TQ ? sW[Ra] : 0.f, wb = Rb / 4 < TQ ? sW[Rb] : 0.f;
        float v[4] = {wa * fmaxf(acc[0], 0.f), wa * fmaxf(acc[1], 0.f), wb * fmaxf(acc[2], 0.f),
                      wb * fmaxf(acc[3], 0.f)};
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // the token's 4 indexer heads
          v[e] += __shfl_xor_sync(0xffffffffu, v[e], 4);
          v[e] += __shfl_xor_sync(0xffffffffu, v[e], 8);
        }
        if (qr % 4 == 0) {
          if (Ra / 4 < TQ) {
            sStu[(Ra / 4) * 8 + 2 * qc] = v[0];
            sStu[(Ra / 4) * 8 + 2 * qc + 1] = v[1];
          }
          if (Rb / 4 < TQ) {
            sStu[(Rb / 4) * 8 + 2 * qc] = v[2];
            sStu[(Rb / 4) * 8 + 2 * qc + 1] = v[3];
          }
        }
      }
      __syncthreads();
      // per (token, block): fold into the token's sums (8 lanes per token)
      if (warp < (TQ * 8 + 31) / 32) {
        const int b = p0 / 4 + kl_blk;
        const bool live = kl_thr && kl_t >= 0 && b < (kl_t >> 2);
        const float m = live ? sMass[kl_tok * 8 + kl_blk] : 0.f;
        const float s = live ? sStu[kl_tok * 8 + kl_blk] : -INFINITY;
        if (kl_thr) sMass[kl_tok * 8 + kl_blk] = 0.f;
        if (live && a.teacher) a.teacher[(long long)(row0 + kl_tok) * a.ld + b] = m;
        float fM = m, fA = m > 0.f ? m * logf(m) : 0.f, fB = live ? m * s : 0.f, smax = s;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          fM += __shfl_xor_sync(0xffffffffu, fM, o);
          fA += __shfl_xor_sync(0xffffffffu, fA, o);
          fB += __shfl_xor_sync(0xffffffffu, fB, o);
          smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
        }
        float fs = live ? expf(s - smax) : 0.f;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) fs += __shfl_xor_sync(0xffffffffu, fs, o);
        if (kl_blk == 0 && smax > -INFINITY) {
          accM += fM;
          accA += fA;
          accB += fB;
          if (smax > lmax) {
            lsum = lsum * exp((double)(lmax - smax)) + fs;
            lmax = smax;
          } else {
            lsum += (double)fs * exp((double)(smax - lmax));
          }
        }
      }
    }
    cp_async_wait<0>();
    __syncthreads();
    if (kl_thr && kl_blk == 0 && kl_t >= 0) {
      float kl = 0.f;
      if ((kl_t >> 2) > 0 && accM > 0.0)
        kl = (float)(accA / accM - log(accM) - accB / accM + lmax + log(lsum));
      a.kl[row0 + kl_tok] = kl;
      sM[kl_tok] = (float)accM;
    }
    __syncthreads();
    if (a.teacher) {  // the masses written above, divided by their total
      for (int i = 0; i < TQ; ++i) {
        const int t = sT[i];
        if (t < 4) continue;
        const float inv = sM[i] > 0.f ? 1.f / sM[i] : 0.f;
        float* row = a.teacher + (long long)(row0 + i) * a.ld;
        for (int b = tid; b < (t >> 2); b += DL_THREADS) row[b] *= inv;
      }
    }
    __syncthreads();
  }
}

template <int D, int DI>
cudaError_t run_distill(const DistillArgs& a, cudaStream_t s) {
  const DlLayout L(D, DI, a.TQ, a.Hq, a.Hkv);
  cudaError_t e = set_smem_once(distill_kl_kernel<D, DI>, L.total);
  if (e != cudaSuccess) return e;
  const int grid = (a.num_q + a.TQ - 1) / a.TQ;
  distill_kl_kernel<D, DI><<<grid, DL_THREADS, L.total, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_distill(const Geometry& g, const void* q, const void* k_pool, const void* idx_q,
                           const void* idx_w, const void* kcomp, float* kl, float* lse,
                           float* teacher, int64_t ld, cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  DistillArgs a;
  a.q = static_cast<const bf16*>(q);
  a.k_pool = static_cast<const bf16*>(k_pool);
  a.idx_q = static_cast<const bf16*>(idx_q);
  a.idx_w = static_cast<const bf16*>(idx_w);
  a.kcomp = static_cast<const bf16*>(kcomp);
  a.q_seq = g.q_seq;
  a.q_pos = g.q_pos;
  a.page_table = g.page_table;
  a.num_q = g.num_q;
  a.batch = g.batch;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.max_pos = g.max_pos;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.G = g.G;
  a.TQ = 256 / g.Hq < 16 ? 256 / g.Hq : 16;
  a.scale_log2 = g.scale_log2;
  a.kl = kl;
  a.lse = lse;
  a.teacher = teacher;
  a.ld = ld;
  a.err = g.err;
  switch (g.D * 1000 + g.Di) {
    case 64032: return run_distill<64, 32>(a, s);
    case 64064: return run_distill<64, 64>(a, s);
    case 64128: return run_distill<64, 128>(a, s);
    case 128032: return run_distill<128, 32>(a, s);
    case 128064: return run_distill<128, 64>(a, s);
    default: return run_distill<128, 128>(a, s);
  }
}

}  // namespace qsa
