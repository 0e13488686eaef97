// Steps (d)+(e): expansion of the selected micro-blocks to token positions and sparse core
// attention over them.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "A million-token window
// with a selective view": the winning micro-blocks are expanded back to token positions and core
// attention runs there only.  Every query head of a token shares the token's selection (one shared
// indexer key head); head h reads key/value head h / (Hq/Hkv).
//
// B200 design.  The work is a gather: per query token up to 513 blocks x 4 positions x Hkv x D x
// 2 (K,V) x 2 bytes = 4.2 MB at Hkv = 4, D = 128, for 8 flop/byte -- HBM-bound, far from the tensor
// roofline.  One CTA serves one query row (or one split of it).
//
// sparse_attn_sw_kernel (Hq/Hkv <= 8, every configuration measured here):
//  * all threads first turn the CTA's selection entries into physical rows (page table, causal
//    clip at t); a producer warp then issues one 4 KB bulk copy (TMA engine, cp.async.bulk) per
//    selected block of K and of V -- a block's 4 positions x all KV heads are contiguous in a
//    page -- into a 3-stage ring, with block slots skewed by 16 bytes so that ldmatrix is
//    conflict-free;
//  * consumer warp (g, slice) takes KV head g and every NSLC-th group of 4 blocks; the MMAs run
//    swap-AB: positions are the M = 16 rows of mma.m16n8k16 and the group's query heads are N = 8,
//    so no MMA row is padding; online softmax in fp32 (exp2 domain), P in bf16 into P*V;
//  * the slices of each KV head merge through shared memory, every consumer thread taking 4 head
//    dims of one query head; split-K partials (decode) go to the workspace, and the last split of
//    the row to finish (a per-row counter) bulk-copies them into its idle stage ring and merges
//    them by log-sum-exp.
//
// sparse_attn_kernel (Hq/Hkv > 8): one bulk copy per position row (Hkv x D x 2 bytes), the query
// heads of a group as the MMA rows, and split-K partials merged by combine_kernel.
#include "common.cuh"
#include "internal.h"
#include "attn_sw.cuh"

namespace qsa {
namespace {
template <int D, int HKV>
struct AttnCfg {
  static constexpr int NCW = 8;                // consumer warps
  static constexpr int NSLC = NCW / HKV;       // chunk slices per kv head
  static constexpr int NBS = 4 * NSLC;         // selected blocks per stage
  static constexpr int ROWS = NBS * 4;         // position rows per stage
  static constexpr int ROWB = HKV * D * 2;     // bytes of one position row (all kv heads)
  static constexpr int PITCH = ROWB + 16;      // skewed shared-memory pitch
  static constexpr int KVB = ROWS * PITCH;     // one tensor, one stage
  static constexpr int STAGE = 2 * KVB;
  static constexpr int NST = (3 * STAGE <= 200 * 1024) ? 3 : 2;
  static constexpr int MERGE = NCW * 16 * (D + 2) * 4;
  static constexpr int BIG = (NST * STAGE > MERGE) ? NST * STAGE : MERGE;
  static constexpr int POS_OFF = BIG;
  static constexpr int BAR_OFF = POS_OFF + NST * ROWS * 4;
  static constexpr int TOTAL = BAR_OFF + 2 * NST * 8 + 16;
  static constexpr int THREADS = (NCW + 1) * 32;
};

template <int D, int HKV>
__global__ void __launch_bounds__(AttnCfg<D, HKV>::THREADS, 1) sparse_attn_kernel(AttnArgs a) {
  chain_wait();
  chain_release();
  using C = AttnCfg<D, HKV>;
  extern __shared__ __align__(128) uint8_t smem[];
  int* sPos = reinterpret_cast<int*>(smem + C::POS_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::NST;
  const uint32_t sbase = smem_addr(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x, split = blockIdx.y;

  // ---- row validation (uniform over the CTA)
  const int seq = a.q_seq[row];
  const int t = a.q_pos[row];
  bool ok = seq >= 0 && seq < a.batch && t >= 0 && t / 64 < a.max_pages;
  int n = ok ? a.n_sel[row] : 0;
  if (n < 0 || n > a.sel_stride) {
    if (tid == 0) flag_error(a.err, QSA_DEVERR_SEL);
    n = max(0, min(n, a.sel_stride));
  }
  if (!ok) {
    if (tid == 0) flag_error(a.err, (seq < 0 || seq >= a.batch) ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);
    n = 0;
  }
  const int blo = (int)((long long)n * split / a.splits);
  const int bhi = (int)((long long)n * (split + 1) / a.splits);
  const int nstages = (bhi - blo + C::NBS - 1) / C::NBS;

  if (tid == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NCW);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == C::NCW) {
    // ================================================================ producer
    constexpr int RPL = (C::ROWS + 31) / 32;  // rows per lane
    const int32_t* selrow = a.sel + (long long)row * a.sel_stride;
    const int32_t* ptab = a.page_table + (long long)(ok ? seq : 0) * a.max_pages;
    int it = 0;
    for (; it < nstages; ++it) {
      const int st = it % C::NST;
      if (it >= C::NST && !mbar_wait(&empty[st], ((it / C::NST) - 1) & 1, a.err)) break;
      const uint32_t kdst = sbase + st * C::STAGE;
      const uint32_t vdst = kdst + C::KVB;
      long long srow[RPL];
      int nvalid = 0;
#pragma unroll
      for (int u = 0; u < RPL; ++u) {
        const int rr = lane + 32 * u;
        srow[u] = -1;
        if (rr < C::ROWS) {
          const int si = blo + it * C::NBS + (rr >> 2);
          int pos = -1;
          if (si < bhi) {
            const int b = selrow[si];
            if (b < 0 || b > t / 4) {
              flag_error(a.err, QSA_DEVERR_SEL);
            } else {
              const int p = 4 * b + (rr & 3);
              if (p <= t) {
                const int page = ptab[p >> 6];
                if (page < 0 || page >= a.num_pages) {
                  flag_error(a.err, QSA_DEVERR_PAGE);
                } else {
                  pos = p;
                  srow[u] = (long long)page * 64 + (p & 63);
                }
              }
            }
          }
          sPos[st * C::ROWS + rr] = pos;
          if (pos < 0) {  // masked row: zeros keep 0 * V finite
            uint4 z = make_uint4(0, 0, 0, 0);
            uint4* kz = reinterpret_cast<uint4*>(smem + st * C::STAGE + rr * C::PITCH);
            uint4* vz = reinterpret_cast<uint4*>(smem + st * C::STAGE + C::KVB + rr * C::PITCH);
#pragma unroll 4
            for (int i = 0; i < C::ROWB / 16; ++i) {
              kz[i] = z;
              vz[i] = z;
            }
          } else {
            ++nvalid;
          }
        }
      }
      const int total = warp_sum_i(nvalid);
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)total * C::ROWB * 2);
      __syncwarp();
#pragma unroll
      for (int u = 0; u < RPL; ++u) {
        const int rr = lane + 32 * u;
        if (srow[u] >= 0) {
          const long long off = srow[u] * (HKV * D);
          bulk_g2s(kdst + rr * C::PITCH, a.k_pool + off, C::ROWB, &full[st]);
          bulk_g2s(vdst + rr * C::PITCH, a.v_pool + off, C::ROWB, &full[st]);
        }
      }
    }
    drain_stages(full, it, C::NST, lane, a.err);
    return;
  }

  // ================================================================== consumers
  const int g = warp % HKV;
  const int slc = warp / HKV;
  const int qr = lane >> 2, qc = lane & 3;
  const int G = a.G;
  uint32_t qf[D / 16][4];
  {
    const bf16* qrow = a.q + (long long)row * a.Hq * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int d0 = ks * 16 + 2 * qc;
      const bool h0 = ok && qr < G, h1 = ok && qr + 8 < G;
      const uint32_t* p0 = reinterpret_cast<const uint32_t*>(qrow + (long long)(g * G + qr) * D + d0);
      const uint32_t* p1 = reinterpret_cast<const uint32_t*>(qrow + (long long)(g * G + qr + 8) * D + d0);
      qf[ks][0] = h0 ? p0[0] : 0u;
      qf[ks][1] = h1 ? p1[0] : 0u;
      qf[ks][2] = h0 ? p0[4] : 0u;
      qf[ks][3] = h1 ? p1[4] : 0u;
    }
  }
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float NEG = -INFINITY;

  for (int it = 0; it < nstages; ++it) {
    const int st = it % C::NST;
    if (!mbar_wait(&full[st], (it / C::NST) & 1, a.err)) break;
    const int* pp = sPos + st * C::ROWS + slc * 16;
    const int pa0 = pp[2 * qc], pa1 = pp[2 * qc + 1], pb0 = pp[8 + 2 * qc], pb1 = pp[9 + 2 * qc];
    const bool any = __any_sync(0xffffffffu, pa0 >= 0 || pa1 >= 0 || pb0 >= 0 || pb1 >= 0);
    if (any) {
      const uint32_t kb = sbase + st * C::STAGE + (slc * 16) * C::PITCH + g * D * 2;
      const uint32_t vb = kb + C::KVB;
      float s[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t kf[4];
        ldsm_x4(kf, kb + ((lane & 7) + ((lane >> 4) << 3)) * C::PITCH + ((ks * 2 + ((lane >> 3) & 1)) << 4));
        mma_bf16_16816(s[0], qf[ks], kf[0], kf[1]);
        mma_bf16_16816(s[1], qf[ks], kf[2], kf[3]);
      }
      // mask + scale (log2 domain)
      float x[2][4];
      x[0][0] = pa0 >= 0 ? s[0][0] * a.scale_log2 : NEG;
      x[0][1] = pa1 >= 0 ? s[0][1] * a.scale_log2 : NEG;
      x[0][2] = pa0 >= 0 ? s[0][2] * a.scale_log2 : NEG;
      x[0][3] = pa1 >= 0 ? s[0][3] * a.scale_log2 : NEG;
      x[1][0] = pb0 >= 0 ? s[1][0] * a.scale_log2 : NEG;
      x[1][1] = pb1 >= 0 ? s[1][1] * a.scale_log2 : NEG;
      x[1][2] = pb0 >= 0 ? s[1][2] * a.scale_log2 : NEG;
      x[1][3] = pb1 >= 0 ? s[1][3] * a.scale_log2 : NEG;
      float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = mn0 == NEG ? 1.f : exp2f(m0 - mn0);
      const float al1 = mn1 == NEG ? 1.f : exp2f(m1 - mn1);
      float p[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        p[nt][0] = mn0 == NEG ? 0.f : exp2f(x[nt][0] - mn0);
        p[nt][1] = mn0 == NEG ? 0.f : exp2f(x[nt][1] - mn0);
        p[nt][2] = mn1 == NEG ? 0.f : exp2f(x[nt][2] - mn1);
        p[nt][3] = mn1 == NEG ? 0.f : exp2f(x[nt][3] - mn1);
      }
      l0 = l0 * al0 + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
      l1 = l1 * al1 + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al0;
        o[i][2] *= al1;
        o[i][3] *= al1;
      }
      uint32_t pf[4];
      pf[0] = pack_bf16(p[0][0], p[0][1]);
      pf[1] = pack_bf16(p[0][2], p[0][3]);
      pf[2] = pack_bf16(p[1][0], p[1][1]);
      pf[3] = pack_bf16(p[1][2], p[1][3]);
#pragma unroll
      for (int dn = 0; dn < D / 16; ++dn) {
        uint32_t vf[4];
        ldsm_x4_t(vf, vb + ((lane & 7) + (((lane >> 3) & 1) << 3)) * C::PITCH + ((dn * 2 + (lane >> 4)) << 4));
        mma_bf16_16816(o[2 * dn], pf, vf[0], vf[1]);
        mma_bf16_16816(o[2 * dn + 1], pf, vf[2], vf[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- merge the slices of each head group (named barrier over the consumer warps only)
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  asm volatile("bar.sync 1, %0;\n" ::"n"(C::NCW * 32));
  float* sO = reinterpret_cast<float*>(smem) + warp * 16 * (D + 2);  // [16][D] then m[16], l[16]
  float* sM = sO + 16 * D;
  float* sL = sM + 16;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const int d = i * 8 + 2 * qc;
    sO[qr * D + d] = o[i][0];
    sO[qr * D + d + 1] = o[i][1];
    sO[(qr + 8) * D + d] = o[i][2];
    sO[(qr + 8) * D + d + 1] = o[i][3];
  }
  if (qc == 0) {
    sM[qr] = m0;
    sM[qr + 8] = m1;
    sL[qr] = l0;
    sL[qr + 8] = l1;
  }
  asm volatile("bar.sync 1, %0;\n" ::"n"(C::NCW * 32));
  const int total = HKV * G * D;
  for (int idx = tid; idx < total; idx += C::NCW * 32) {
    const int gg = idx / (G * D);
    const int h = (idx / D) % G;
    const int d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < C::NSLC; ++s) {
      const float* base = reinterpret_cast<float*>(smem) + (s * HKV + gg) * 16 * (D + 2);
      M = fmaxf(M, base[16 * D + h]);
    }
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int s = 0; s < C::NSLC; ++s) {
        const float* base = reinterpret_cast<float*>(smem) + (s * HKV + gg) * 16 * (D + 2);
        const float ms = base[16 * D + h];
        if (ms != -INFINITY) {
          const float f = exp2f(ms - M);
          L += base[16 * D + 16 + h] * f;
          O += base[h * D + d] * f;
        }
      }
    }
    const int hq = gg * G + h;
    const float res = L > 0.f ? O / L : 0.f;
    const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
    if (a.splits == 1) {
      a.out[((long long)row * a.Hq + hq) * D + d] = __float2bfloat16_rn(res);
      if (a.lse && d == 0) a.lse[(long long)row * a.Hq + hq] = lse2 * 0.69314718055994531f;
    } else {
      const long long pi = ((long long)row * a.splits + split) * a.Hq + hq;
      a.part_o[pi * D + d] = res;
      if (d == 0) a.part_lse[pi] = lse2;
    }
  }
}

template <int D, int HKV, int SLC>
__global__ void __launch_bounds__(SwCfg<D, HKV, SLC>::THREADS, 1) sparse_attn_sw_kernel(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  chain_wait();
  chain_release();
  sparse_attn_sw_body<D, HKV, SLC>(a, blockIdx.x, blockIdx.y, smem);
}

// Zero n counters, as a chained launch (a memset between two chained kernels would break the
// chain).  It waits for the previous grid first: that grid may still count on the same words.
__global__ void zero_u32_kernel(uint32_t* __restrict__ p, int n) {
  chain_wait();
  chain_release();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0;
}

// Merge split-K partials: out = sum_s 2^(lse_s - L) o_s, L = log2 sum_s 2^lse_s.
__global__ void combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                               int splits, int Hq, int D, bf16* __restrict__ out, float* lse) {
  const int row = blockIdx.x, h = blockIdx.y;
  const long long base = (long long)row * splits * Hq + h;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, part_lse[base + (long long)s * Hq]);
  float L = 0.f;
  if (M != -INFINITY)
    for (int s = 0; s < splits; ++s) {
      const float v = part_lse[base + (long long)s * Hq];
      if (v != -INFINITY) L += exp2f(v - M);
    }
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    if (L > 0.f)
      for (int s = 0; s < splits; ++s) {
        const float v = part_lse[base + (long long)s * Hq];
        if (v != -INFINITY) acc += exp2f(v - M) * part_o[(base + (long long)s * Hq) * D + d];
      }
    out[((long long)row * Hq + h) * D + d] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
  }
  if (lse && threadIdx.x == 0)
    lse[(long long)row * Hq + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

template <int D, int HKV>
cudaError_t run_sparse(const AttnArgs& a, int splits, cudaStream_t s) {
  if (a.G <= 8) {
    constexpr int SLC = kSwSlices<HKV>;
    using C = SwCfg<D, HKV, SLC>;
    cudaError_t e = set_smem_once(sparse_attn_sw_kernel<D, HKV, SLC>, C::TOTAL);
    if (e != cudaSuccess) return e;
    return launch_chained(sparse_attn_sw_kernel<D, HKV, SLC>, dim3(a.num_q, splits), dim3(C::THREADS), C::TOTAL, s,
                          a);
  }
  using C = AttnCfg<D, HKV>;
  cudaError_t e = set_smem_once(sparse_attn_kernel<D, HKV>, C::TOTAL);
  if (e != cudaSuccess) return e;
  return launch_chained(sparse_attn_kernel<D, HKV>, dim3(a.num_q, splits), dim3(C::THREADS), C::TOTAL, s, a);
}

}  // namespace

int resolve_sparse_splits(const Geometry& g, int requested) {
  if (requested > 0) return requested > 64 ? 64 : requested;
  if (g.num_q <= 0) return 1;
  int s = num_sms() / g.num_q;
  if (s < 1) s = 1;
  const int max_useful = (g.topk + 1 + 7) / 8;
  if (s > max_useful) s = max_useful;
  if (s > 64) s = 64;
  return s;
}

// Split-K workspace: partial outputs fp32 [num_q, splits, Hq, D], their log2-sum-exp
// [num_q, splits, Hq], and (swap-AB kernel, Hq/Hkv <= 8) per-row arrival counters [num_q].
size_t sparse_decode_workspace_bytes(const Geometry& g, int splits) {
  if (splits <= 1) return 0;
  const size_t n = (size_t)g.num_q * splits * g.Hq;
  return ((n * g.D * 4 + 255) / 256) * 256 + ((n * 4 + 255) / 256) * 256 +
         (((size_t)g.num_q * 4 + 255) / 256) * 256;
}

cudaError_t launch_combine(const Geometry& g, const float* part_o, const float* part_lse,
                           int splits, void* out, float* lse, cudaStream_t s) {
  combine_kernel<<<dim3(g.num_q, g.Hq), g.D, 0, s>>>(part_o, part_lse, splits, g.Hq, g.D,
                                                     static_cast<bf16*>(out), lse);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const Geometry& g, const void* q, const void* k_pool,
                               const void* v_pool, const int32_t* sel, const int32_t* n_sel,
                               int sel_stride, void* out, float* lse, int splits, void* ws,
                               cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  AttnArgs a;
  a.q = static_cast<const bf16*>(q);
  a.k_pool = static_cast<const bf16*>(k_pool);
  a.v_pool = static_cast<const bf16*>(v_pool);
  a.sel = sel;
  a.n_sel = n_sel;
  a.sel_stride = sel_stride;
  a.q_seq = g.q_seq;
  a.q_pos = g.q_pos;
  a.page_table = g.page_table;
  a.num_q = g.num_q;
  a.batch = g.batch;
  a.max_pages = g.max_pages;
  a.num_pages = g.num_pages;
  a.Hq = g.Hq;
  a.G = g.G;
  a.scale_log2 = g.scale_log2;
  a.out = static_cast<bf16*>(out);
  a.lse = lse;
  a.splits = splits;
  a.err = g.err;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  a.arrivals = nullptr;
  a.coop = 0;
  a.departures = nullptr;
  if (splits > 1) {
    const size_t n = (size_t)g.num_q * splits * g.Hq;
    a.part_o = static_cast<float*>(ws);
    a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ((n * g.D * 4 + 255) / 256) * 256);
    a.arrivals = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.part_lse) + ((n * 4 + 255) / 256) * 256);
    if (g.G <= 8) {  // the swap-AB kernel merges its splits itself, counting arrivals from zero
      cudaError_t e = launch_chained(zero_u32_kernel, dim3((g.num_q + 255) / 256), dim3(256), 0, s, a.arrivals,
                                     g.num_q);
      if (e != cudaSuccess) return e;
    }
  }
  cudaError_t e;
#define QSA_SPARSE_CASE(DD, HH) \
  if (g.D == DD && g.Hkv == HH) e = run_sparse<DD, HH>(a, splits, s); else
  QSA_SPARSE_CASE(64, 1)
  QSA_SPARSE_CASE(64, 2)
  QSA_SPARSE_CASE(64, 4)
  QSA_SPARSE_CASE(64, 8)
  QSA_SPARSE_CASE(128, 1)
  QSA_SPARSE_CASE(128, 2)
  QSA_SPARSE_CASE(128, 4)
  QSA_SPARSE_CASE(128, 8)
  e = cudaErrorInvalidValue;
#undef QSA_SPARSE_CASE
  if (e != cudaSuccess || splits == 1 || g.G <= 8) return e;
  return launch_combine(g, a.part_o, a.part_lse, splits, out, lse, s);
}

}  // namespace qsa
