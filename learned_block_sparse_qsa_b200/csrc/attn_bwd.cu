// Backward pass of the sparse core attention (steps (d)+(e) with the selection held fixed).
//
// Article "Qwen's million-token window has a 2,048-token keyhole", section "The indexer is trained,
// not bolted on": after the dense warm-up QSA selected the blocks core attention uses while the
// indexer and the backbone trained together, so gradients flow through the sparse attention; the
// top-k choice itself has no gradient.  For one query row and head h (key/value head g):
//     a = softmax_p(scale q_h . k_p) over the row's attended positions,  o_h = sum_p a_p v_p,
//     dv_p += a_p do_h,  dz_p = a_p (do_h . v_p - do_h . o_h),
//     dq_h = scale sum_p dz_p k_p,  dk_p += scale dz_p q_h.
// The forward's log-sum-exp gives a_p without a second softmax pass.
//
// One CTA per query row, 8 warps, Hq/Hkv <= 8: warp (g, slice) takes KV head g and every
// NSLC-th group of 4 selected blocks, in the swap-AB layout of the forward -- the 16 positions of
// 4 blocks are the M rows of mma.m16n8k16 and the group's query heads are N = 8:
//   S^T = K Q^T and dA^T = V dO^T (m16n8k16, K and V from shared memory by ldmatrix);
//   P^T and dS^T in registers;  dQ^T += K^T dS^T (m16n8k16, dS^T transposed with movmatrix);
//   dV = P^T dO and dK = scale dS^T Q (m16n8k8, 8 heads deep), added to fp32 gradient pools with
//   16-byte vector atomics (lane pairs swap halves of their fragments first), since every row
//   that selected a block contributes to its keys and values.
// Selected blocks stream through a 2-stage cp.async ring, a block's 4 positions of all KV heads
// being one contiguous 4 KB run of its page (16-byte skewed slots, as in the forward).
#include "common.cuh"
#include "internal.h"

namespace qsa {
namespace {

constexpr int BW_MAXSEL = 520;

template <int D, int HKV>
struct BwCfg {
  static constexpr int NCW = 8;
  static constexpr int NSLC = NCW / HKV;
  static constexpr int NBS = 4 * NSLC;      // blocks per stage (4 per warp slice)
  static constexpr int ROWB = HKV * D * 2;  // one position row, all KV heads
  static constexpr int BLKB = 4 * ROWB;
  static constexpr int BPITCH = BLKB + 16;
  static constexpr int KVB = NBS * BPITCH;
  static constexpr int STAGE = 2 * KVB;
  static constexpr int NST = 2;
  static constexpr int MERGE = NCW * 8 * D * 4;  // dQ^T slices [warp][8 heads][D]
  static constexpr int BIG = NST * STAGE > MERGE ? NST * STAGE : MERGE;
  static constexpr int ROW_OFF = BIG;                         // int [BW_MAXSEL]
  static constexpr int BLK_OFF = ROW_OFF + BW_MAXSEL * 4;     // int [BW_MAXSEL]
  static constexpr int HEAD_OFF = BLK_OFF + BW_MAXSEL * 4;    // float [2][128]: lse2, D_h
  static constexpr int TOTAL = HEAD_OFF + 2 * 128 * 4;
  static constexpr int THREADS = NCW * 32;
};

struct BwArgs {
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
  float scale, scale_log2;
  const bf16* out;
  const float* lse;
  const bf16* dout;
  float* dq;
  float* dk;
  float* dv;
  int32_t* err;
};

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void mma_bf16_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

// Add a fragment's pair of pairs as one 16-byte reduction: the m16n8 accumulator gives lane
// (qr, qc) dims 2qc, 2qc+1 of rows qr (c0, c1) and qr + 8 (c2, c3); lanes qc and qc ^ 1 swap
// halves so that the even lane adds dims 2qc..2qc+3 of row qr and the odd lane dims
// 2qc-2..2qc+1 of row qr + 8.  base_a / base_b: the rows' addresses at dim 0 of this n-tile
// (nullptr: that row is not added); 16-byte aligned.
__device__ __forceinline__ void red_add_quad(float* base_a, float* base_b, const float (&c)[4], float scale, int qc) {
  const bool odd = qc & 1;
  const float s0 = odd ? c[0] : c[2], s1 = odd ? c[1] : c[3];  // what the partner needs
  const float r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
  float* dst = odd ? base_b : base_a;
  if (!dst) return;
  const float4 v = odd ? make_float4(r0 * scale, r1 * scale, c[2] * scale, c[3] * scale)
                       : make_float4(c[0] * scale, c[1] * scale, r0 * scale, r1 * scale);
  atomicAdd(reinterpret_cast<float4*>(dst + 2 * (qc & ~1)), v);
}

template <int D, int HKV>
__global__ void __launch_bounds__(BwCfg<D, HKV>::THREADS, 1) sparse_attn_bwd_kernel(BwArgs a) {
  using C = BwCfg<D, HKV>;
  extern __shared__ __align__(128) uint8_t smem[];
  int* sRow = reinterpret_cast<int*>(smem + C::ROW_OFF);
  int* sBlk = reinterpret_cast<int*>(smem + C::BLK_OFF);
  float* sLse2 = reinterpret_cast<float*>(smem + C::HEAD_OFF);
  float* sDh = sLse2 + 128;
  const uint32_t sbase = smem_addr(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x;
  const int G = a.G;

  const int seq = a.q_seq[row];
  const int t = a.q_pos[row];
  const bool ok = seq >= 0 && seq < a.batch && t >= 0 && t / 64 < a.max_pages;
  int n = ok ? a.n_sel[row] : 0;
  if (n < 0 || n > a.sel_stride || n > BW_MAXSEL) {
    if (tid == 0) flag_error(a.err, QSA_DEVERR_SEL);
    n = max(0, min(min(n, a.sel_stride), BW_MAXSEL));
  }
  if (!ok && tid == 0) flag_error(a.err, (seq < 0 || seq >= a.batch) ? QSA_DEVERR_SEQ : QSA_DEVERR_POS);

  // selected blocks -> physical rows; per-head log2-sum-exp and D_h = do_h . o_h
  {
    const int32_t* selrow = a.sel + (long long)row * a.sel_stride;
    const int32_t* ptab = a.page_table + (long long)(ok ? seq : 0) * a.max_pages;
    for (int i = tid; i < n; i += C::THREADS) {
      const int b = selrow[i];
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
    for (int h = warp; h < a.Hq; h += C::NCW) {
      float s = 0.f;
      if (ok) {
        const bf16* op = a.out + ((long long)row * a.Hq + h) * D;
        const bf16* gp = a.dout + ((long long)row * a.Hq + h) * D;
        for (int d = lane; d < D; d += 32) s += __bfloat162float(op[d]) * __bfloat162float(gp[d]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) {
        sDh[h] = s;
        sLse2[h] = ok ? a.lse[(long long)row * a.Hq + h] * 1.4426950408889634f : INFINITY;
      }
    }
  }
  __syncthreads();

  const int nstages = (n + C::NBS - 1) / C::NBS;
  auto load = [&](int it, int st) {
    const uint32_t kb = sbase + st * C::STAGE;
    for (int i = tid; i < C::NBS * (C::BLKB / 16); i += C::THREADS) {
      const int j = i / (C::BLKB / 16), c = i % (C::BLKB / 16);
      const int bi = it * C::NBS + j;
      const int rb = bi < n ? sRow[bi] : -1;
      const int nvalid = rb >= 0 ? min(4, t - 4 * sBlk[bi] + 1) : 0;
      const bool valid = c / (C::ROWB / 16) < nvalid;  // rows past t (tail clip) zero-filled
      const long long off = (long long)(rb < 0 ? 0 : rb) * (HKV * D) + c * 8;
      cp_async16(kb + j * C::BPITCH + c * 16, a.k_pool + off, valid);
      cp_async16(kb + C::KVB + j * C::BPITCH + c * 16, a.v_pool + off, valid);
    }
  };

  const int g = warp % HKV, slc = warp / HKV;
  const int qr = lane >> 2, qc = lane & 3;
  const bool hv = ok && qr < G;  // this lane's B-operand head exists
  // Q^T and dO^T as m16n8k16 B operands (k = head dims, n = heads), Q and dO as m16n8k8 B
  // operands (k = heads 2qc, 2qc+1; n = head dim n0 + qr)
  uint32_t qb[D / 16][2], gb[D / 16][2], qn[D / 8], gn[D / 8];
  {
    const uint32_t* qp = reinterpret_cast<const uint32_t*>(a.q + ((long long)row * a.Hq + g * G + qr) * D);
    const uint32_t* gp = reinterpret_cast<const uint32_t*>(a.dout + ((long long)row * a.Hq + g * G + qr) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qb[ks][0] = hv ? qp[ks * 8 + qc] : 0u;
      qb[ks][1] = hv ? qp[ks * 8 + 4 + qc] : 0u;
      gb[ks][0] = hv ? gp[ks * 8 + qc] : 0u;
      gb[ks][1] = hv ? gp[ks * 8 + 4 + qc] : 0u;
    }
    const int h0 = 2 * qc, h1 = 2 * qc + 1;
    const bf16* q0 = a.q + ((long long)row * a.Hq + g * G + h0) * D;
    const bf16* q1 = a.q + ((long long)row * a.Hq + g * G + h1) * D;
    const bf16* g0 = a.dout + ((long long)row * a.Hq + g * G + h0) * D;
    const bf16* g1 = a.dout + ((long long)row * a.Hq + g * G + h1) * D;
    const bool v0 = ok && h0 < G, v1 = ok && h1 < G;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int d = nt * 8 + qr;
      __nv_bfloat162 x, y;
      x.x = v0 ? q0[d] : __float2bfloat16_rn(0.f);
      x.y = v1 ? q1[d] : __float2bfloat16_rn(0.f);
      y.x = v0 ? g0[d] : __float2bfloat16_rn(0.f);
      y.y = v1 ? g1[d] : __float2bfloat16_rn(0.f);
      qn[nt] = *reinterpret_cast<uint32_t*>(&x);
      gn[nt] = *reinterpret_cast<uint32_t*>(&y);
    }
  }
  const int h0 = 2 * qc, h1 = 2 * qc + 1;
  const float l0 = h0 < G ? sLse2[g * G + h0] : INFINITY, l1 = h1 < G ? sLse2[g * G + h1] : INFINITY;
  const float d0 = h0 < G ? sDh[g * G + h0] : 0.f, d1 = h1 < G ? sDh[g * G + h1] : 0.f;

  float dqt[D / 16][4];  // dQ^T: rows = head dims (16 per m-tile), cols = heads
#pragma unroll
  for (int i = 0; i < D / 16; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dqt[i][e] = 0.f;
  auto row_off = [&](int mrow) { return (4 * slc + (mrow & 3)) * C::BPITCH + (mrow >> 2) * C::ROWB; };
  const int kr = (lane & 7) + (((lane >> 3) & 1) << 3);
  const int vr = (lane & 7) + ((lane >> 4) << 3);
  const uint32_t koff = row_off(kr) + g * D * 2 + ((lane >> 4) << 4);         // K (and V) rows
  const uint32_t toff = row_off(vr) + g * D * 2 + (((lane >> 3) & 1) << 4);  // K^T (trans)

  if (nstages > 0) load(0, 0);
  cp_async_commit();
  for (int it = 0; it < nstages; ++it) {
    cp_async_wait<0>();
    __syncthreads();
    if (it + 1 < nstages) load(it + 1, (it + 1) & 1);
    cp_async_commit();
    const int st = it & 1;
    // positions of this warp's MMA rows qr and qr + 8: slot 4*slc + (r&3), row r>>2 of the block
    auto pos_of = [&](int r) {
      const int bi = it * C::NBS + 4 * slc + (r & 3);
      if (bi >= n || sRow[bi] < 0) return -1;
      const int p = 4 * sBlk[bi] + (r >> 2);
      return p <= t ? p : -1;
    };
    const int pa = pos_of(qr), pb = pos_of(qr + 8);
    if (!__any_sync(0xffffffffu, pa >= 0 || pb >= 0)) continue;
    const uint32_t kbase = sbase + st * C::STAGE, vbase = kbase + C::KVB;
    float s[4] = {0.f, 0.f, 0.f, 0.f}, da[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t kf[4], vf[4];
      ldsm_x4(kf, kbase + koff + ks * 32);
      mma_bf16_16816(s, kf, qb[ks][0], qb[ks][1]);
      ldsm_x4(vf, vbase + koff + ks * 32);
      mma_bf16_16816(da, vf, gb[ks][0], gb[ks][1]);
    }
    // s/da[0]=(row qr, head 2qc) [1]=(qr, 2qc+1) [2]=(qr+8, 2qc) [3]=(qr+8, 2qc+1)
    const float p0 = pa >= 0 ? exp2f(s[0] * a.scale_log2 - l0) : 0.f;
    const float p1 = pa >= 0 ? exp2f(s[1] * a.scale_log2 - l1) : 0.f;
    const float p2 = pb >= 0 ? exp2f(s[2] * a.scale_log2 - l0) : 0.f;
    const float p3 = pb >= 0 ? exp2f(s[3] * a.scale_log2 - l1) : 0.f;
    const float s0 = p0 * (da[0] - d0), s1 = p1 * (da[1] - d1);
    const float s2 = p2 * (da[2] - d0), s3 = p3 * (da[3] - d1);
    // dQ^T += K^T dS^T
    const uint32_t db0 = movmatrix_t(pack_bf16(s0, s1));
    const uint32_t db1 = movmatrix_t(pack_bf16(s2, s3));
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t kt[4];
      ldsm_x4_t(kt, kbase + toff + mt * 32);
      mma_bf16_16816(dqt[mt], kt, db0, db1);
    }
    // dV = P^T dO and dK = scale dS^T Q, 8 head dims at a time, added to the fp32 pools
    const uint32_t pa0 = pack_bf16(p0, p1), pa1 = pack_bf16(p2, p3);
    const uint32_t sa0 = pack_bf16(s0, s1), sa1 = pack_bf16(s2, s3);
    const long long ra = pa >= 0 ? ((long long)(sRow[it * C::NBS + 4 * slc + (qr & 3)] + (qr >> 2)) * HKV + g) * D : -1;
    const long long rb = pb >= 0 ? ((long long)(sRow[it * C::NBS + 4 * slc + ((qr + 8) & 3)] + ((qr + 8) >> 2)) * HKV + g) * D : -1;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      float cv[4] = {0.f, 0.f, 0.f, 0.f}, ck[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16_1688(cv, pa0, pa1, gn[nt]);
      mma_bf16_1688(ck, sa0, sa1, qn[nt]);
      red_add_quad(ra >= 0 ? a.dv + ra + nt * 8 : nullptr, rb >= 0 ? a.dv + rb + nt * 8 : nullptr, cv, 1.f, qc);
      red_add_quad(ra >= 0 ? a.dk + ra + nt * 8 : nullptr, rb >= 0 ? a.dk + rb + nt * 8 : nullptr, ck, a.scale, qc);
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  // the slices of each KV head: dQ^T partials through shared memory, then dq = scale * sum
  float* sQ = reinterpret_cast<float*>(smem) + warp * 8 * D;  // [8 heads][D]
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int d = mt * 16 + qr;
    sQ[(2 * qc) * D + d] = dqt[mt][0];
    sQ[(2 * qc + 1) * D + d] = dqt[mt][1];
    sQ[(2 * qc) * D + d + 8] = dqt[mt][2];
    sQ[(2 * qc + 1) * D + d + 8] = dqt[mt][3];
  }
  __syncthreads();
  const float* sm = reinterpret_cast<const float*>(smem);
  for (int e = tid; e < HKV * G * D; e += C::THREADS) {
    const int hq = e / D, d = e % D;
    const int gg = hq / G, h = hq % G;
    float acc = 0.f;
#pragma unroll
    for (int sl = 0; sl < C::NSLC; ++sl) acc += sm[((sl * HKV + gg) * 8 + h) * D + d];
    a.dq[((long long)row * a.Hq + hq) * D + d] = ok ? acc * a.scale : 0.f;
  }
}

template <int D, int HKV>
cudaError_t run_bwd(const BwArgs& a, cudaStream_t s) {
  using C = BwCfg<D, HKV>;
  cudaError_t e = set_smem_once(sparse_attn_bwd_kernel<D, HKV>, C::TOTAL);
  if (e != cudaSuccess) return e;
  sparse_attn_bwd_kernel<D, HKV><<<a.num_q, C::THREADS, C::TOTAL, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn_bwd(const Geometry& g, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* sel, const int32_t* n_sel,
                                   const void* out, const float* lse, const void* dout, float* dq,
                                   float* dk_pool, float* dv_pool, cudaStream_t s) {
  if (g.num_q == 0) return cudaSuccess;
  if (g.G > 8 || g.Hq > 128) return cudaErrorNotSupported;
  BwArgs a;
  a.q = static_cast<const bf16*>(q);
  a.k_pool = static_cast<const bf16*>(k_pool);
  a.v_pool = static_cast<const bf16*>(v_pool);
  a.sel = sel;
  a.n_sel = n_sel;
  a.sel_stride = g.topk + 1;
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
  a.scale = g.scale_log2 * 0.69314718055994531f;
  a.out = static_cast<const bf16*>(out);
  a.lse = lse;
  a.dout = static_cast<const bf16*>(dout);
  a.dq = dq;
  a.dk = dk_pool;
  a.dv = dv_pool;
  a.err = g.err;
#define QSA_BWD_CASE(DD, HH) \
  if (g.D == DD && g.Hkv == HH) return run_bwd<DD, HH>(a, s);
  QSA_BWD_CASE(64, 1)
  QSA_BWD_CASE(64, 2)
  QSA_BWD_CASE(64, 4)
  QSA_BWD_CASE(64, 8)
  QSA_BWD_CASE(128, 1)
  QSA_BWD_CASE(128, 2)
  QSA_BWD_CASE(128, 4)
  QSA_BWD_CASE(128, 8)
#undef QSA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace qsa
