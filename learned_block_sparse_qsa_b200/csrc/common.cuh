// Device helpers for the libqsa kernels (sm_100a): bf16 packing, legacy-MMA fragments,
// cp.async, mbarriers with bounded waits, and 1-D bulk copies (TMA engine, no tensor map).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "../../include/qsa.h"

namespace qsa {

typedef __nv_bfloat16 bf16;

// Roughly one second at B200 clocks: a wait that lasts longer than this is a bug, so it is
// reported through the error flag instead of hanging the GPU.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Opt a kernel into more than 48 KB of dynamic shared memory, once per (kernel, device), on the
// host.  Done at the first launch so that later launches -- possibly inside a stream capture --
// issue no attribute calls.  Kernels are told apart by address (several share one signature).
inline cudaError_t set_smem_once(const void* kernel, int bytes) {
  struct Entry {
    const void* k;
    unsigned long long devs;
  };
  static Entry table[64];
  static int used = 0;
  static std::mutex lock;  // host threads may launch on their own streams concurrently
  std::lock_guard<std::mutex> guard(lock);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  int i = 0;
  while (i < used && table[i].k != kernel) ++i;
  if (i < used && (table[i].devs & bit)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (i == used && used < 64) table[used++] = Entry{kernel, 0};
  if (i < used) table[i].devs |= bit;
  return cudaSuccess;
}
template <typename Kernel>
inline cudaError_t set_smem_once(Kernel* k, int bytes) {
  return set_smem_once(reinterpret_cast<const void*>(k), bytes);
}

// Programmatic dependent launch.  The chained kernels of a layer step (compress, indexer,
// selection, attention) are launched with launch_chained(): such a kernel may be scheduled while
// the previous kernel in the stream is still running, so that its launch and start-up overlap the
// previous kernel's tail.  Every kernel launched that way calls chain_wait() as its first
// statement, before it reads or writes any global memory, and then chain_release().
//   chain_wait():    returns once the previous grid in the stream has completed and its memory
//                    operations are visible (a no-op for an ordinary launch).  Because every
//                    chained kernel waits before it can complete, completion is transitive along
//                    the chain.
//   chain_release(): lets the next chained grid be scheduled (its CTAs then sit in their own
//                    chain_wait() until this grid completes).  Called after the wait, so at most
//                    two grids of a chain are resident at a time, and a waiting grid holds no
//                    tensor memory (every allocation comes after the wait).  A kernel that does
//                    not call it releases the next grid when it exits.
__device__ __forceinline__ void chain_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void chain_release() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Barrier over `n` threads (a multiple of 32) under id `id` (1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void flag_error(int32_t* err, uint32_t bits) {
  if (err) atomicOr(err, (int32_t)bits);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------- legacy tensor-core MMA
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// ---------------------------------------------------------------- cp.async (16-byte)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // src-size 0 zero-fills the destination
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---------------------------------------------------------------- mbarrier + bulk copy
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: true when the phase completed, false (and QSA_DEVERR_TIMEOUT) after the limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* err,
                                          long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) {
      flag_error(err, QSA_DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// Global -> shared bulk copy on the TMA engine; bytes and both addresses multiples of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------- ordering keys
// Monotone map of fp32 onto uint32 (larger float -> larger integer); -0 is folded onto +0 by
// the caller so that equal scores compare equal.
__device__ __forceinline__ uint32_t f32_to_ordered(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_f32(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}
// Candidate key: score major, then LOWER block index first.  Keys of distinct blocks differ;
// 0 never occurs for a finite score and marks an empty slot.
__device__ __forceinline__ unsigned long long make_key(float score, uint32_t block) {
  score = __fadd_rn(score, 0.0f);  // -0 + +0 = +0: equal scores get equal keys
  return ((unsigned long long)f32_to_ordered(score) << 32) | (0xFFFFFFFFu - block);
}
__device__ __forceinline__ uint32_t key_block(unsigned long long k) {
  return 0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull);
}
__device__ __forceinline__ float key_score(unsigned long long k) {
  return ordered_to_f32((uint32_t)(k >> 32));
}

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace qsa
