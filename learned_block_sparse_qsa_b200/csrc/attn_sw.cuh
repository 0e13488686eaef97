// Swap-AB sparse attention (Hq/Hkv <= 8) as a CTA-level body: shared by the standalone kernel
// (attn.cu) and the fused decode step (decode_step.cu).  See attn.cu for the design.
#pragma once
#include "common.cuh"
#include "internal.h"

namespace qsa {
namespace {

struct AttnArgs {
  const bf16* q;
  const bf16* k_pool;
  const bf16* v_pool;
  const int32_t* sel;
  const int32_t* n_sel;
  int sel_stride;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int num_q, batch, max_pages, num_pages, Hq, G;
  float scale_log2;
  bf16* out;
  float* lse;
  float* part_o;
  float* part_lse;
  int splits;
  uint32_t* arrivals;  // split-K: per-row count of finished splits (zeroed before the launch)
  // Cooperative combine (only when every split of a row is resident at once, as in a cooperative
  // launch with one split per CTA): each split waits for all of its row's partials, then merges
  // the heads h = split (mod splits); `departures` counts the splits done reading, and the last
  // one sets both counters back to zero.  0 / nullptr: the last split merges every head.
  int coop;
  uint32_t* departures;
  int32_t* err;
};


// The producer warp leaves only after the last (up to nst) stages it posted have landed: in the
// normal course they already have, and after a wait that ran out (already flagged) this is the
// bounded wait for the bulk copies still in flight into this CTA's shared memory.
__device__ __forceinline__ void drain_stages(uint64_t* full, int posted, int nst, int lane, int32_t* err) {
  if (lane != 0) return;
  for (int j = posted > nst ? posted - nst : 0; j < posted; ++j) mbar_wait(&full[j % nst], (j / nst) & 1, err);
}

// Barrier over the first NTHREADS threads of the block (id 2; id 1 is the consumers' own).
template <int NTHREADS>
__device__ __forceinline__ void sw_cta_sync() {
  asm volatile("bar.sync 2, %0;\n" ::"n"(NTHREADS) : "memory");
}

// ------------------------------------------------------------------------------------------------
// Swap-AB form for Hq/Hkv <= 8 (the article's 32 query heads over 4 KV heads): positions are the
// M=16 rows of mma.m16n8k16 and the (up to) 8 query heads of a KV head are N=8, so no MMA row is
// padding; P is transposed in registers with movmatrix for the P*V product, which computes O^T
// (head dims x heads).  The producer first turns the CTA's whole slice of the selection into
// physical row bases in shared memory (one pass, all lanes), so no dependent global load sits
// between two stage issues.

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

constexpr int kMaxSel = 520;  // >= topk + 1
// Consumer warps per KV head; a stage holds 4 blocks (16 positions) per consumer warp, so fewer
// slices mean smaller stages and more of the shared-memory ring in flight.
template <int HKV>
constexpr int kSwSlices = HKV >= 4 ? 2 : 8 / HKV;

template <int D, int HKV, int SLC>
struct SwCfg {
  static constexpr int NSLC = SLC;          // consumer warps per KV head
  static constexpr int NCW = HKV * SLC;
  static constexpr int NBS = 4 * NSLC;      // blocks per stage: 4 (= one 16-position chunk) per slice
  static constexpr int ROWB = HKV * D * 2;  // one position row, all KV heads
  static constexpr int BLKB = 4 * ROWB;     // one block: 4 contiguous rows
  static constexpr int BPITCH = BLKB + 16;  // block slots skewed by 16 bytes
  static constexpr int KVB = NBS * BPITCH;
  static constexpr int STAGE = 2 * KVB;
  static constexpr int NST = (200 * 1024) / STAGE > 8 ? 8 : (200 * 1024) / STAGE;
  static constexpr int MERGE = NCW * (8 * D + 16) * 4;
  static constexpr int BIG = (NST * STAGE > MERGE) ? NST * STAGE : MERGE;
  static constexpr int POS_OFF = BIG;
  static constexpr int ROW_OFF = POS_OFF + NST * NBS * 4 * 4;
  static constexpr int BLK_OFF = ROW_OFF + kMaxSel * 4;
  static constexpr int BAR_OFF = BLK_OFF + kMaxSel * 4;
  static constexpr int TOTAL = BAR_OFF + (2 * NST + 1) * 8 + 8;  // full, empty, combine barriers
  static constexpr int THREADS = (NCW + 1) * 32;
  static_assert(NBS <= 32, "one producer lane per block slot");
};

// Stage layout: block slot j (0..NBS-1) holds the 4 rows of one selected block, K at
// j*BPITCH and V at KVB + j*BPITCH.  Consumer warp `slc` owns slots 4*slc .. 4*slc+3; its MMA row
// r (0..15) is row r>>2 of slot 4*slc + (r&3), so an 8-row ldmatrix reads 4 slots (distinct 16-byte
// skews) x 2 rows: at most a 2-way bank conflict, while every full block arrives in one 4 KB copy.
// The kernel body for the CTA of (row, split), run by threads 0 .. SwCfg::THREADS-1 of the
// calling block (its CTA-wide syncs are a named barrier over exactly those threads, so a larger
// block can run it with its other warps elsewhere).  smem: SwCfg::TOTAL bytes, 128-byte aligned.
template <int D, int HKV, int SLC>
__device__ __forceinline__ void sparse_attn_sw_body(const AttnArgs& a, const int row, const int split,
                                                    uint8_t* smem) {
  using C = SwCfg<D, HKV, SLC>;
  int* sPos = reinterpret_cast<int*>(smem + C::POS_OFF);  // [stage][slot*4 + row-in-block]
  int* sRow = reinterpret_cast<int*>(smem + C::ROW_OFF);  // page*64 + (b%16)*4, or -1
  int* sBlk = reinterpret_cast<int*>(smem + C::BLK_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::NST;
  uint64_t* cbar = empty + C::NST;  // split-K combine: the row's partials arriving
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int seq = a.q_seq[row];
  const int t = a.q_pos[row];
  const bool ok = seq >= 0 && seq < a.batch && t >= 0 && t / 64 < a.max_pages;
  int n = ok ? a.n_sel[row] : 0;
  if (n < 0 || n > a.sel_stride || n > kMaxSel) {
    if (tid == 0) flag_error(a.err, QSA_DEVERR_SEL);
    n = max(0, min(min(n, a.sel_stride), kMaxSel));
  }
  if (!ok && tid == 0) flag_error(a.err, (seq < 0 || seq >= a.batch) ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);
  const int blo = (int)((long long)n * split / a.splits);
  const int bhi = (int)((long long)n * (split + 1) / a.splits);
  const int nblk = bhi - blo;
  const int nstages = (nblk + C::NBS - 1) / C::NBS;

  if (tid == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NCW);
    }
    mbar_init(cbar, 1);
    mbar_fence_init();
  }
  {  // every thread: one round of (selection entry -> page table) loads for the CTA's slice
    const int32_t* selrow = a.sel + (long long)row * a.sel_stride;
    const int32_t* ptab = a.page_table + (long long)(ok ? seq : 0) * a.max_pages;
    for (int i = tid; i < nblk; i += C::THREADS) {
      const int b = selrow[blo + i];
      int rb = -1;
      if (b < 0 || b > t / 4) {
        flag_error(a.err, QSA_DEVERR_SEL);
      } else {
        const int page = ptab[b >> 4];
        if (page < 0 || page >= a.num_pages) flag_error(a.err, QSA_DEVERR_PAGE);
        else rb = page * 64 + (b & 15) * 4;
      }
      sRow[i] = rb;
      sBlk[i] = b;
    }
  }
  sw_cta_sync<C::THREADS>();

  if (warp == C::NCW) {
    // ================================================================ producer
    int it = 0;
    for (; it < nstages; ++it) {
      const int st = it % C::NST;
      if (it >= C::NST && !mbar_wait(&empty[st], ((it / C::NST) - 1) & 1, a.err)) break;
      const uint32_t kdst = sbase + st * C::STAGE + lane * C::BPITCH;
      const uint32_t vdst = kdst + C::KVB;
      // lane j < NBS serves block slot j: rows valid = 4 (whole block), 1..3 (tail), or 0
      int nvalid = 0, rb = -1;
      if (lane < C::NBS) {
        const int i = it * C::NBS + lane;
        int b = 0;
        if (i < nblk && sRow[i] >= 0) {
          rb = sRow[i];
          b = sBlk[i];
          nvalid = min(4, t - 4 * b + 1);
        }
        int* pp = sPos + (st * C::NBS + lane) * 4;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          pp[r] = r < nvalid ? 4 * b + r : -1;
          if (r >= nvalid) {  // masked row: zeros keep 0 * V finite
            const uint4 z = make_uint4(0, 0, 0, 0);
            uint4* kz = reinterpret_cast<uint4*>(smem + st * C::STAGE + lane * C::BPITCH + r * C::ROWB);
            uint4* vz = reinterpret_cast<uint4*>(smem + st * C::STAGE + C::KVB + lane * C::BPITCH + r * C::ROWB);
#pragma unroll 4
            for (int j = 0; j < C::ROWB / 16; ++j) {
              kz[j] = z;
              vz[j] = z;
            }
          }
        }
      }
      const int total = warp_sum_i(nvalid);
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)total * C::ROWB * 2);
      __syncwarp();
      if (nvalid > 0) {
        const long long off = (long long)rb * (HKV * D);
        if (nvalid == 4) {
          bulk_g2s(kdst, a.k_pool + off, C::BLKB, &full[st]);
          bulk_g2s(vdst, a.v_pool + off, C::BLKB, &full[st]);
        } else {
          for (int r = 0; r < nvalid; ++r) {
            bulk_g2s(kdst + r * C::ROWB, a.k_pool + off + (long long)r * HKV * D, C::ROWB, &full[st]);
            bulk_g2s(vdst + r * C::ROWB, a.v_pool + off + (long long)r * HKV * D, C::ROWB, &full[st]);
          }
        }
      }
    }
    drain_stages(full, it, C::NST, lane, a.err);
  } else {
  // ================================================================== consumers
  const int g = warp % HKV;
  const int slc = warp / HKV;
  const int G = a.G;
  const int qr = lane >> 2, qc = lane & 3;
  // Q^T as the B operand: b0 = Q[head qr][16ks + 2qc ..], b1 = Q[head qr][16ks + 8 + 2qc ..]
  uint32_t qb[D / 16][2];
  {
    const bool hv = ok && qr < G;
    const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.q + ((long long)row * a.Hq + g * G + qr) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qb[ks][0] = hv ? qp[ks * 8 + qc] : 0u;
      qb[ks][1] = hv ? qp[ks * 8 + 4 + qc] : 0u;
    }
  }
  float o[D / 16][4];  // O^T: rows = head dims (16 per m-tile), cols = heads
#pragma unroll
  for (int i = 0; i < D / 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2qc, 2qc+1
  const float NEG = -INFINITY;
  // this lane's ldmatrix row: MMA row ((lane&7) + 8*sel) -> slot (row&3), row-in-block (row>>2)
  auto row_off = [&](int mrow) { return (4 * slc + (mrow & 3)) * C::BPITCH + (mrow >> 2) * C::ROWB; };
  const int kr = (lane & 7) + (((lane >> 3) & 1) << 3);  // K: A-operand row of this lane
  const int vr = (lane & 7) + ((lane >> 4) << 3);         // V^T: k (= position) row of this lane
  const uint32_t koff = row_off(kr) + g * D * 2 + ((lane >> 4) << 4);
  const uint32_t voff = row_off(vr) + g * D * 2 + (((lane >> 3) & 1) << 4);

  for (int it = 0; it < nstages; ++it) {
    const int st = it % C::NST;
    if (!mbar_wait(&full[st], (it / C::NST) & 1, a.err)) break;
    const int* pp = sPos + (st * C::NBS + 4 * slc) * 4;
    const int pa = pp[(qr & 3) * 4 + (qr >> 2)];              // MMA row qr
    const int pb = pp[((qr + 8) & 3) * 4 + ((qr + 8) >> 2)];  // MMA row qr + 8
    if (__any_sync(0xffffffffu, pa >= 0 || pb >= 0)) {
      const uint32_t kb = sbase + st * C::STAGE;
      const uint32_t vb = kb + C::KVB;
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t kf[4];
        ldsm_x4(kf, kb + koff + ks * 32);
        mma_bf16_16816(s, kf, qb[ks][0], qb[ks][1]);
      }
      // s[0]=(row qr, head 2qc) s[1]=(qr, 2qc+1) s[2]=(qr+8, 2qc) s[3]=(qr+8, 2qc+1)
      const float x0 = pa >= 0 ? s[0] * a.scale_log2 : NEG;
      const float x1 = pa >= 0 ? s[1] * a.scale_log2 : NEG;
      const float x2 = pb >= 0 ? s[2] * a.scale_log2 : NEG;
      const float x3 = pb >= 0 ? s[3] * a.scale_log2 : NEG;
      float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = mn0 == NEG ? 1.f : exp2f(m0 - mn0);
      const float al1 = mn1 == NEG ? 1.f : exp2f(m1 - mn1);
      const float p0 = mn0 == NEG ? 0.f : exp2f(x0 - mn0);
      const float p1 = mn1 == NEG ? 0.f : exp2f(x1 - mn1);
      const float p2 = mn0 == NEG ? 0.f : exp2f(x2 - mn0);
      const float p3 = mn1 == NEG ? 0.f : exp2f(x3 - mn1);
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int i = 0; i < D / 16; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al1;
        o[i][2] *= al0;
        o[i][3] *= al1;
      }
      // P^T as the B operand (k = MMA row/position, n = head): transpose the two 8x8 blocks
      const uint32_t pb0 = movmatrix_t(pack_bf16(p0, p1));
      const uint32_t pb1 = movmatrix_t(pack_bf16(p2, p3));
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t vf[4];
        ldsm_x4_t(vf, vb + voff + mt * 32);
        mma_bf16_16816(o[mt], vf, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- merge slices of each KV head through shared memory (consumer warps only)
#pragma unroll
  for (int o2 = 4; o2 < 32; o2 <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o2);
  }
  asm volatile("bar.sync 1, %0;\n" ::"n"(C::NCW * 32));
  float* sO = reinterpret_cast<float*>(smem) + warp * (8 * D + 16);  // [8 heads][D], m[8], l[8]
  float* sM = sO + 8 * D;
  float* sL = sM + 8;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int d = mt * 16 + qr;
    sO[(2 * qc) * D + d] = o[mt][0];
    sO[(2 * qc + 1) * D + d] = o[mt][1];
    sO[(2 * qc) * D + d + 8] = o[mt][2];
    sO[(2 * qc + 1) * D + d + 8] = o[mt][3];
  }
  if (qr == 0) {
    sM[2 * qc] = m0;
    sM[2 * qc + 1] = m1;
    sL[2 * qc] = l0;
    sL[2 * qc + 1] = l1;
  }
  asm volatile("bar.sync 1, %0;\n" ::"n"(C::NCW * 32));
  // every consumer thread merges 4 head dims of one query head at a time: the slices' m and l
  // give the weights, then one 16-byte read per slice and one 8- or 16-byte store
  {
    constexpr int D4 = D / 4;
    const int lg = __ffs(G) - 1;  // G is a power of two
    const int n4 = HKV * G * D4;
    const float* sm = reinterpret_cast<const float*>(smem);
#pragma unroll 4
    for (int e = tid; e < n4; e += C::NCW * 32) {
      const int hq = e / D4, d = (e % D4) * 4;
      const int gg = hq >> lg, h = hq & (G - 1);
      float ms[C::NSLC], f[C::NSLC];
      float M = -INFINITY, L = 0.f;
#pragma unroll
      for (int sl = 0; sl < C::NSLC; ++sl) {
        ms[sl] = sm[(sl * HKV + gg) * (8 * D + 16) + 8 * D + h];
        M = fmaxf(M, ms[sl]);
      }
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int sl = 0; sl < C::NSLC; ++sl) {
        const float* base = sm + (sl * HKV + gg) * (8 * D + 16);
        f[sl] = (M != -INFINITY && ms[sl] != -INFINITY) ? exp2f(ms[sl] - M) : 0.f;
        L += base[8 * D + 8 + h] * f[sl];
        const float4 o = *reinterpret_cast<const float4*>(base + h * D + d);
        O.x = fmaf(o.x, f[sl], O.x);
        O.y = fmaf(o.y, f[sl], O.y);
        O.z = fmaf(o.z, f[sl], O.z);
        O.w = fmaf(o.w, f[sl], O.w);
      }
      const float inv = L > 0.f ? 1.0f / L : 0.f;
      const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
      O.x *= inv;
      O.y *= inv;
      O.z *= inv;
      O.w *= inv;
      if (a.splits == 1) {
        uint2 packed;
        packed.x = pack_bf16(O.x, O.y);
        packed.y = pack_bf16(O.z, O.w);
        *reinterpret_cast<uint2*>(a.out + ((long long)row * a.Hq + hq) * D + d) = packed;
        if (d == 0 && a.lse) a.lse[(long long)row * a.Hq + hq] = lse2 * 0.69314718055994531f;
      } else {
        const long long pi = ((long long)row * a.splits + split) * a.Hq + hq;
        *reinterpret_cast<float4*>(a.part_o + pi * D + d) = O;
        if (d == 0) a.part_lse[pi] = lse2;
      }
    }
  }
  }  // consumers

  if (a.splits > 1 && a.coop) {
    __threadfence();
    sw_cta_sync<C::THREADS>();
    if (tid == 0) {
      atomicAdd(&a.arrivals[row], 1u);
      const volatile uint32_t* ar = a.arrivals + row;
      const long long t0 = clock64();
      while (*ar < (uint32_t)a.splits) {
        if (clock64() - t0 > kWaitLimitCycles) {
          flag_error(a.err, QSA_DEVERR_TIMEOUT);
          break;
        }
      }
      __threadfence();
    }
    sw_cta_sync<C::THREADS>();
    const int S = a.splits, Hq = a.Hq;
    const long long b0 = (long long)row * S * Hq;  // partial index of (split 0, head 0)
    const int nh = (Hq - split + S - 1) / S;       // this split's heads: split, split + S, ...
    constexpr int D4 = D / 4;
    const long long step = (long long)Hq * D / 4;  // float4s between splits
    // the first PRE partials of this thread's first output group are loaded before anything else,
    // so that their latency overlaps the weights' computation
    constexpr int PRE = 8;
    float4 pre[PRE];
    {
      const int e = tid;
      if (e < nh * D4) {
        const float4* src = reinterpret_cast<const float4*>(a.part_o + (b0 + split + (e / D4) * S) * D + (e % D4) * 4);
#pragma unroll
        for (int j = 0; j < PRE; ++j) pre[j] = j < S ? __ldcg(src + j * step) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    // the heads' S log-sum-exps, loaded at once into the idle stage ring, then turned into the
    // last-split merge's weights (same values, same order: the output is bit-identical)
    float* wn = reinterpret_cast<float*>(smem);    // [nh][S]
    for (int i = tid; i < nh * S; i += C::THREADS) {
      const int hi = i / S, sp = i % S;
      wn[i] = __ldcg(a.part_lse + b0 + (long long)sp * Hq + split + hi * S);
    }
    sw_cta_sync<C::THREADS>();
    if (tid < nh) {
      float* w = wn + tid * S;
      float M = -INFINITY, L = 0.f;
      for (int sp = 0; sp < S; ++sp) M = fmaxf(M, w[sp]);
      for (int sp = 0; sp < S; ++sp) {
        const float e = (M != -INFINITY && w[sp] != -INFINITY) ? exp2f(w[sp] - M) : 0.f;
        w[sp] = e;
        L += e;
      }
      const float inv = L > 0.f ? 1.0f / L : 0.f;
      for (int sp = 0; sp < S; ++sp) w[sp] *= inv;
      if (a.lse)
        a.lse[(long long)row * Hq + split + tid * S] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
    sw_cta_sync<C::THREADS>();
    for (int e = tid; e < nh * D4; e += C::THREADS) {
      const int hi = e / D4, hq = split + hi * S, d = (e % D4) * 4;
      const float* w = wn + hi * S;
      const float4* src = reinterpret_cast<const float4*>(a.part_o + (b0 + hq) * D + d);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      int sp = 0;
      if (e == tid) {  // the preloaded group
#pragma unroll
        for (int j = 0; j < PRE; ++j) {
          if (j < S) {
            acc.x = fmaf(w[j], pre[j].x, acc.x);
            acc.y = fmaf(w[j], pre[j].y, acc.y);
            acc.z = fmaf(w[j], pre[j].z, acc.z);
            acc.w = fmaf(w[j], pre[j].w, acc.w);
          }
        }
        sp = S < PRE ? S : PRE;
      }
      for (; sp < S; ++sp) {
        const float4 p = __ldcg(src + sp * step);
        acc.x = fmaf(w[sp], p.x, acc.x);
        acc.y = fmaf(w[sp], p.y, acc.y);
        acc.z = fmaf(w[sp], p.z, acc.z);
        acc.w = fmaf(w[sp], p.w, acc.w);
      }
      uint2 packed;
      packed.x = pack_bf16(acc.x, acc.y);
      packed.y = pack_bf16(acc.z, acc.w);
      *reinterpret_cast<uint2*>(a.out + ((long long)row * Hq + hq) * D + d) = packed;
    }
    sw_cta_sync<C::THREADS>();
    if (tid == 0 && atomicAdd(&a.departures[row], 1u) == (uint32_t)S - 1u) {
      a.arrivals[row] = 0u;  // every split of the row has read its partials
      a.departures[row] = 0u;
    }
  } else if (a.splits > 1) {
    // the last split of the row to finish merges all of the row's partials (log-sum-exp weights)
    __shared__ int s_last;
    __threadfence();
    sw_cta_sync<C::THREADS>();
    if (tid == 0) s_last = atomicAdd(&a.arrivals[row], 1u) == (uint32_t)a.splits - 1u;
    sw_cta_sync<C::THREADS>();
    if (s_last) {
      __threadfence();
      const int S = a.splits, Hq = a.Hq;
      const long long b0 = (long long)row * S * Hq;  // partial index of (split 0, head 0)
      const int nv = Hq * D / 4;                      // float4 groups of one split's output
      // the row's partials are contiguous ([S][Hq][D] fp32): when they fit in the idle stage
      // ring, bulk copies bring them in while the weights below are computed
      const uint32_t pbytes = (uint32_t)S * Hq * D * 4;
      const bool staged = (size_t)pbytes + (size_t)Hq * S * 4 <= (size_t)C::BIG;
      if (staged && tid == 0) {
        // generic-proxy partials of the other splits (ordered by their fences and the counter),
        // and this CTA's earlier shared-memory use, before the async-proxy copies
        asm volatile("fence.proxy.async;\n" ::: "memory");
        mbar_arrive_expect_tx(cbar, pbytes);
        const uint32_t per = (uint32_t)Hq * D * 4;
        for (int sp = 0; sp < S; ++sp)
          bulk_g2s(sbase + sp * per, a.part_o + (b0 + (long long)sp * Hq) * D, per, cbar);
      }
      // weights 2^(lse_s - M) / sum into shared memory [Hq][S]: every (head, split) log-sum-exp
      // is loaded at once, then one thread per head reduces its S values
      float* wn = reinterpret_cast<float*>(smem + (staged ? pbytes : 0u));
      for (int p = tid; p < Hq * S; p += C::THREADS) {
        const int hq = p / S, sp = p % S;
        wn[p] = __ldcg(a.part_lse + b0 + (long long)sp * Hq + hq);
      }
      sw_cta_sync<C::THREADS>();
      if (tid < Hq) {
        float* w = wn + tid * S;
        float M = -INFINITY, L = 0.f;
        for (int sp = 0; sp < S; ++sp) M = fmaxf(M, w[sp]);
        for (int sp = 0; sp < S; ++sp) {
          const float e = (M != -INFINITY && w[sp] != -INFINITY) ? exp2f(w[sp] - M) : 0.f;
          w[sp] = e;
          L += e;
        }
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        for (int sp = 0; sp < S; ++sp) w[sp] *= inv;
        if (a.lse)
          a.lse[(long long)row * Hq + tid] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
      }
      sw_cta_sync<C::THREADS>();
      bf16* orow = a.out + (long long)row * Hq * D;
      if (staged) {
        if (!mbar_wait(cbar, 0, a.err)) {
          mbar_wait(cbar, 0, a.err);  // ran out: wait once more, bounded, for the copies in flight
        } else {
          const float4* ps = reinterpret_cast<const float4*>(smem);
          for (int v = tid; v < nv; v += C::THREADS) {
            const float* w = wn + (v * 4 / D) * S;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int sp = 0; sp < S; ++sp) {
              const float4 p = ps[sp * nv + v];
              acc.x = fmaf(w[sp], p.x, acc.x);
              acc.y = fmaf(w[sp], p.y, acc.y);
              acc.z = fmaf(w[sp], p.z, acc.z);
              acc.w = fmaf(w[sp], p.w, acc.w);
            }
            uint2 packed;
            packed.x = pack_bf16(acc.x, acc.y);
            packed.y = pack_bf16(acc.z, acc.w);
            *reinterpret_cast<uint2*>(orow + (long long)v * 4) = packed;
          }
        }
      } else {
        // outputs: each thread owns up to 4 float4 groups of head dims and walks the splits
        // once, so that 4 independent 16-byte loads per split (12 with the unrolling) are in flight
        constexpr int VPT = 4;
        const long long sstride = (long long)Hq * D / 4;  // float4s between splits
        const float4* part4 = reinterpret_cast<const float4*>(a.part_o) + b0 * D / 4;
        for (int v0 = tid; v0 < nv; v0 += VPT * C::THREADS) {
          float4 acc[VPT];
          int hqv[VPT];
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            hqv[j] = (v0 + j * C::THREADS) * 4 / D;
          }
#pragma unroll 3
          for (int sp = 0; sp < S; ++sp) {
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
              const int v = v0 + j * C::THREADS;
              if (v < nv) {
                const float w = wn[hqv[j] * S + sp];
                const float4 p = __ldcg(part4 + sp * sstride + v);
                acc[j].x = fmaf(w, p.x, acc[j].x);
                acc[j].y = fmaf(w, p.y, acc[j].y);
                acc[j].z = fmaf(w, p.z, acc[j].z);
                acc[j].w = fmaf(w, p.w, acc[j].w);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            const int v = v0 + j * C::THREADS;
            if (v < nv) {
              uint2 packed;
              packed.x = pack_bf16(acc[j].x, acc[j].y);
              packed.y = pack_bf16(acc[j].z, acc[j].w);
              *reinterpret_cast<uint2*>(orow + (long long)v * 4) = packed;
            }
          }
        }
      }
      if (tid == 0) a.arrivals[row] = 0u;
    }
  }
}

}  // namespace
}  // namespace qsa
