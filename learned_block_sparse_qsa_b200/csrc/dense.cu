// The comparison baseline: dense causal paged grouped-query attention over every position <= t.
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "Three speed claims,
// three different experiments": the QSA module's speedups are quoted against paged grouped-query
// attention at one million tokens.  This kernel is that baseline on the same paged pools, so the
// sparse/dense ratio measured here compares two kernels of this library.
//
// The prefill form at head_dim 128 runs on the tensor cores (dense_tc.cu); this file holds the
// mma.sync kernel for the other shapes and the decode form.
// Flash-attention tiling: a CTA owns MR = TQ x G query rows of one KV head (the G query heads of
// TQ consecutive tokens of one sequence), streams the sequence's pages (64 positions) of that KV
// head through a 3-stage cp.async ring, and keeps fp32 online-softmax state in registers.  The
// decode form splits the context across CTAs and merges by log-sum-exp.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace qsa {
namespace {

struct DenseArgs {
  const bf16* q;
  const bf16* k_pool;
  const bf16* v_pool;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* page_table;
  int num_q, batch, max_pages, num_pages, Hq, Hkv, G;
  float scale_log2;
  bf16* out;
  float* lse;
  float* part_o;
  float* part_lse;
  int splits;
  int32_t* err;
};

template <int D>
__device__ __forceinline__ uint32_t swzd(int r, int c) {
  return (uint32_t)(r * (D * 2) + ((c ^ (r & 7)) << 4));
}

constexpr int DN_NST = 3;
// Positions per K/V tile of the small-batch (decode) form: half a page, so that a CTA's ring is
// 48 KB at head_dim 128 and four CTAs share an SM (a whole page: 96 KB, two CTAs, four warps).
constexpr int kDecPT = 32;

template <int D, int MR, int PT>
struct DenseCfg {
  static_assert(PT == 32 || PT == 64, "a tile is a page or half a page");
  static constexpr int WARPS = MR / 16;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int TILE = PT * D * 2;  // one tensor, PT positions of one kv head
  static constexpr int TOTAL = DN_NST * 2 * TILE + 64;
};

template <int D, int MR, int PT>
__global__ void __launch_bounds__(DenseCfg<D, MR, PT>::THREADS) dense_attn_kernel(DenseArgs a) {
  using C = DenseCfg<D, MR, PT>;
  constexpr int CH = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sK = smem_addr(smem);
  const uint32_t sV = sK + DN_NST * C::TILE;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int TQ = MR / G;
  const int row0 = blockIdx.x * TQ;
  const int g = blockIdx.y;
  const int split = blockIdx.z;
  const int qr = lane >> 2, qc = lane & 3;
  // this thread's two M rows
  const int ma = warp * 16 + qr, mb = ma + 8;
  const int rowa = row0 + ma / G, rowb = row0 + mb / G;
  const int ha = ma % G, hb = mb % G;
  int seqa = -1, seqb = -1, ta = -1, tb = -1;
  if (rowa < a.num_q) { seqa = a.q_seq[rowa]; ta = a.q_pos[rowa]; }
  if (rowb < a.num_q) { seqb = a.q_seq[rowb]; tb = a.q_pos[rowb]; }
  auto valid_row = [&](int s, int t) { return s >= 0 && s < a.batch && t >= 0 && t / 64 < a.max_pages; };
  if (tid == 0) {
    for (int i = 0; i < TQ; ++i) {
      const int r = row0 + i;
      if (r >= a.num_q) break;
      if (!valid_row(a.q_seq[r], a.q_pos[r]))
        flag_error(a.err, (a.q_seq[r] < 0 || a.q_seq[r] >= a.batch) ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);
    }
  }
  const bool oka = rowa < a.num_q && valid_row(seqa, ta);
  const bool okb = rowb < a.num_q && valid_row(seqb, tb);

  uint32_t qf[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int d0 = ks * 16 + 2 * qc;
    const uint32_t* pa = reinterpret_cast<const uint32_t*>(a.q + ((long long)rowa * a.Hq + g * G + ha) * D + d0);
    const uint32_t* pb = reinterpret_cast<const uint32_t*>(a.q + ((long long)rowb * a.Hq + g * G + hb) * D + d0);
    qf[ks][0] = oka ? pa[0] : 0u;
    qf[ks][1] = okb ? pb[0] : 0u;
    qf[ks][2] = oka ? pa[4] : 0u;
    qf[ks][3] = okb ? pb[4] : 0u;
  }

  // Segments: rows of the tile that share a sequence share the KV stream.
  unsigned long long done_mask = 0;  // bit i: token i of the tile handled (same in every thread)
  for (;;) {
    int seg = -1, tmax = -1;
    for (int i = 0; i < TQ; ++i) {
      const int r = row0 + i;
      if (r >= a.num_q || ((done_mask >> i) & 1ull)) continue;
      const int s = a.q_seq[r], t = a.q_pos[r];
      if (!valid_row(s, t)) { done_mask |= 1ull << i; continue; }
      if (seg < 0) seg = s;
      if (s == seg) { tmax = max(tmax, t); done_mask |= 1ull << i; }
    }
    if (seg < 0) break;
    const bool acta = oka && seqa == seg, actb = okb && seqb == seg;
    const int ntot = tmax / PT + 1;  // tiles of PT positions up to the segment's last query
    const int p_lo = (int)((long long)ntot * split / a.splits);
    const int p_hi = (int)((long long)ntot * (split + 1) / a.splits);
    const int ntiles = p_hi - p_lo;
    const int32_t* ptab = a.page_table + (long long)seg * a.max_pages;

    auto load = [&](int it, int st) {
      const int p0 = (p_lo + it) * PT;  // first position of the tile
      const int lp = p0 / 64, off = p0 % 64;
      int page = ptab[lp];
      bool ok = page >= 0 && page < a.num_pages;
      if (!ok && tid == 0) flag_error(a.err, QSA_DEVERR_PAGE);
      if (!ok) page = 0;
      for (int i = tid; i < 2 * PT * CH; i += C::THREADS) {
        const int tsr = i / (PT * CH);
        const int rem = i % (PT * CH);
        const int pr = rem / CH, c = rem % CH;
        const bf16* pool = tsr ? a.v_pool : a.k_pool;
        const bf16* src = pool + (((long long)page * 64 + off + pr) * a.Hkv + g) * D + c * 8;
        // positions past the segment's last query may be unwritten cache slots: zero them so
        // that masked probabilities (0) never meet a non-finite value
        cp_async16((tsr ? sV : sK) + st * C::TILE + swzd<D>(pr, c), src, ok && p0 + pr <= tmax);
      }
    };

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const int tla = acta ? ta : -1, tlb = actb ? tb : -1;

    __syncthreads();
    for (int s = 0; s < DN_NST - 1; ++s) {
      if (s < ntiles) load(s, s);
      cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
      cp_async_wait<DN_NST - 2>();
      __syncthreads();
      {
        const int nt = it + DN_NST - 1;
        if (nt < ntiles) load(nt, nt % DN_NST);
        cp_async_commit();
      }
      const int st = it % DN_NST;
      const int pbase = (p_lo + it) * PT;
      if (__any_sync(0xffffffffu, tla >= pbase || tlb >= pbase)) {
        float sc[PT / 8][4];
#pragma unroll
        for (int nt = 0; nt < PT / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
          for (int np = 0; np < PT / 16; ++np) {
            uint32_t kf[4];
            const int pr = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            ldsm_x4(kf, sK + st * C::TILE + swzd<D>(pr, ks * 2 + ((lane >> 3) & 1)));
            mma_bf16_16816(sc[2 * np], qf[ks], kf[0], kf[1]);
            mma_bf16_16816(sc[2 * np + 1], qf[ks], kf[2], kf[3]);
          }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < PT / 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = pbase + nt * 8 + 2 * qc + e;
            sc[nt][e] = p <= tla ? sc[nt][e] * a.scale_log2 : -INFINITY;
            sc[nt][2 + e] = p <= tlb ? sc[nt][2 + e] * a.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, sc[nt][e]);
            mx1 = fmaxf(mx1, sc[nt][2 + e]);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
        const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < PT / 8; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            sc[nt][e] = mn0 == -INFINITY ? 0.f : exp2f(sc[nt][e] - mn0);
            sc[nt][2 + e] = mn1 == -INFINITY ? 0.f : exp2f(sc[nt][2 + e] - mn1);
            rs0 += sc[nt][e];
            rs1 += sc[nt][2 + e];
          }
        }
        l0 = l0 * al0 + rs0;
        l1 = l1 * al1 + rs1;
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          o[i][0] *= al0;
          o[i][1] *= al0;
          o[i][2] *= al1;
          o[i][3] *= al1;
        }
#pragma unroll
        for (int kc = 0; kc < PT / 16; ++kc) {
          uint32_t pf[4];
          pf[0] = pack_bf16(sc[2 * kc][0], sc[2 * kc][1]);
          pf[1] = pack_bf16(sc[2 * kc][2], sc[2 * kc][3]);
          pf[2] = pack_bf16(sc[2 * kc + 1][0], sc[2 * kc + 1][1]);
          pf[3] = pack_bf16(sc[2 * kc + 1][2], sc[2 * kc + 1][3]);
#pragma unroll
          for (int dn = 0; dn < D / 16; ++dn) {
            uint32_t vf[4];
            const int pr = kc * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
            ldsm_x4_t(vf, sV + st * C::TILE + swzd<D>(pr, dn * 2 + (lane >> 4)));
            mma_bf16_16816(o[2 * dn], pf, vf[0], vf[1]);
            mma_bf16_16816(o[2 * dn + 1], pf, vf[2], vf[3]);
          }
        }
      }
    }
    cp_async_wait<0>();
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    // ---- write this segment's rows
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const bool act = half ? actb : acta;
      if (!act) continue;
      const int r = half ? rowb : rowa;
      const int hq = g * G + (half ? hb : ha);
      const float L = half ? l1 : l0, M = half ? m1 : m0;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const float lse2 = L > 0.f ? M + log2f(L) : -INFINITY;
      if (a.splits == 1) {
        bf16* dst = a.out + ((long long)r * a.Hq + hq) * D;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          const int d = i * 8 + 2 * qc;
          const float v0 = (half ? o[i][2] : o[i][0]) * inv, v1 = (half ? o[i][3] : o[i][1]) * inv;
          *reinterpret_cast<__nv_bfloat162*>(dst + d) = __floats2bfloat162_rn(v0, v1);
        }
        if (a.lse && qc == 0) a.lse[(long long)r * a.Hq + hq] = lse2 * 0.69314718055994531f;
      } else {
        const long long pi = ((long long)r * a.splits + split) * a.Hq + hq;
        float* dst = a.part_o + pi * D;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          const int d = i * 8 + 2 * qc;
          dst[d] = (half ? o[i][2] : o[i][0]) * inv;
          dst[d + 1] = (half ? o[i][3] : o[i][1]) * inv;
        }
        if (qc == 0) a.part_lse[pi] = lse2;
      }
    }
  }
}

template <int D, int MR, int PT>
cudaError_t run_dense(const DenseArgs& a, int splits, cudaStream_t s) {
  using C = DenseCfg<D, MR, PT>;
  cudaError_t e = set_smem_once(dense_attn_kernel<D, MR, PT>, C::TOTAL);
  if (e != cudaSuccess) return e;
  const int TQ = MR / a.G;
  const int tiles = (a.num_q + TQ - 1) / TQ;
  dense_attn_kernel<D, MR, PT><<<dim3(tiles, a.Hkv, splits), C::THREADS, C::TOTAL, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

namespace {
// CTAs of the kernel instance that one SM holds at once (its shared memory decides), looked up
// once per process; 1 when the runtime cannot say (no device), with the error cleared.
template <int D, int MR, int PT>
int dense_resident_ctas() {
  static std::atomic<int> cached{0};
  const int c = cached.load(std::memory_order_relaxed);
  if (c > 0) return c;
  using C = DenseCfg<D, MR, PT>;
  int n = 0;
  if (set_smem_once(dense_attn_kernel<D, MR, PT>, C::TOTAL) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dense_attn_kernel<D, MR, PT>, C::THREADS, C::TOTAL) !=
          cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    return 1;
  }
  cached.store(n, std::memory_order_relaxed);
  return n;
}
}  // namespace

// Automatic split count: as many splits as fill the GPU in ONE wave of resident CTAs (a second,
// nearly empty wave would double the time of the whole launch), capped at one page per split.
int resolve_dense_splits(const Geometry& g, int requested) {
  if (requested > 0) return requested;
  const bool small = g.num_q <= 256;
  const int mr = small ? 32 : 64;
  const int tq = mr / g.G;
  const int tiles = (g.num_q + tq - 1) / tq;
  const int ctas = tiles * g.Hkv;
  const int per_sm = g.D == 64 ? (small ? dense_resident_ctas<64, 32, kDecPT>() : dense_resident_ctas<64, 64, 64>())
                               : (small ? dense_resident_ctas<128, 32, kDecPT>() : dense_resident_ctas<128, 64, 64>());
  int s = per_sm * num_sms() / ctas;
  const int pages = g.max_pos / (small ? kDecPT : 64) + 1;  // at most one tile per split
  if (s > pages) s = pages;
  if (s < 1) s = 1;
  return s;
}

size_t dense_decode_workspace_bytes(const Geometry& g, int splits) {
  const size_t n = (size_t)g.num_q * splits * g.Hq;
  return ((n * g.D * 4 + 255) / 256) * 256 + ((n * 4 + 255) / 256) * 256;
}

cudaError_t launch_dense_attn(const Geometry& g, const void* q, const void* k_pool,
                              const void* v_pool, void* out, float* lse, int splits, void* ws,
                              cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  if (splits == 1 && dense_tc_supported(g)) return launch_dense_tc(g, q, k_pool, v_pool, out, lse, s);
  DenseArgs a;
  a.q = static_cast<const bf16*>(q);
  a.k_pool = static_cast<const bf16*>(k_pool);
  a.v_pool = static_cast<const bf16*>(v_pool);
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
  a.scale_log2 = g.scale_log2;
  a.out = static_cast<bf16*>(out);
  a.lse = lse;
  a.splits = splits;
  a.err = g.err;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  if (splits > 1) {
    const size_t n = (size_t)g.num_q * splits * g.Hq;
    a.part_o = static_cast<float*>(ws);
    a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ((n * g.D * 4 + 255) / 256) * 256);
  }
  const bool small = g.num_q <= 256;
  cudaError_t e;
  if (g.D == 64)
    e = small ? run_dense<64, 32, kDecPT>(a, splits, s) : run_dense<64, 64, 64>(a, splits, s);
  else
    e = small ? run_dense<128, 32, kDecPT>(a, splits, s) : run_dense<128, 64, 64>(a, splits, s);
  if (e != cudaSuccess || splits == 1) return e;
  return launch_combine(g, a.part_o, a.part_lse, splits, out, lse, s);
}

}  // namespace qsa
