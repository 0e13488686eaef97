// Exact top-k selection primitives on 64-bit candidate keys (score major, lower block first).
//
// Keys of one query row are unique (they embed the block index), so "the k largest keys" is a
// well-defined set: the article's selection rule (keep the best 512 micro-blocks) under the
// library's tie-break (lower block index wins).
#pragma once
#include "common.cuh"

namespace qsa {

typedef unsigned long long u64;

// Histogram increment with lanes that hit the same bin merged first (same-address shared-memory
// atomics serialise).  Must be called by all 32 lanes of the warp.
__device__ __forceinline__ void hist_add(uint32_t* h, uint32_t bin, bool active) {
  const unsigned am = __ballot_sync(0xffffffffu, active);
  if (active) {
    const unsigned peers = __match_any_sync(am, bin);
    if ((int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&h[bin], (uint32_t)__popc(peers));
  }
}

// One warp: find the `need`-th largest of the `cnt` unique keys in buf[0..cnt) by an MSB-first
// radix select over 8-bit digits, then compact the `need` largest keys into buf[0..need) (order
// unspecified).  Returns the smallest kept key.  hist: 256 words of this warp's shared memory.
// Requires 1 <= need <= cnt.  buf may be global or shared memory.
__device__ __forceinline__ u64 warp_select_compact(u64* buf, int cnt, int need, uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  u64 prefix = 0, mask = 0;
  uint32_t remaining = (uint32_t)need;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) hist[i] = 0;
    __syncwarp();
    for (int base = 0; base < cnt; base += 32) {
      const int i = base + lane;
      const u64 k = i < cnt ? buf[i] : 0ull;
      hist_add(hist, (uint32_t)(k >> shift) & 255u, i < cnt && (k & mask) == prefix);
    }
    __syncwarp();
    // lane l owns bins 255-8l down to 248-8l
    uint32_t c[8], tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      c[j] = hist[255 - 8 * lane - j];
      tot += c[j];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - tot;
    const bool mine = excl < remaining && remaining <= incl;
    int digit = 0;
    uint32_t above = 0;
    if (mine) {
      uint32_t acc = excl;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (acc + c[j] >= remaining) {
          digit = 255 - 8 * lane - j;
          above = acc;
          break;
        }
        acc += c[j];
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, mine);
    const int src = __ffs(bal) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    remaining -= above;
    prefix |= (u64)digit << shift;
    mask |= 0xFFull << shift;
    __syncwarp();
  }
  // prefix is now the need-th largest key; keep every key >= it (exactly `need` keys)
  int w = 0;
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const u64 k = i < cnt ? buf[i] : 0ull;
    const bool keep = i < cnt && k >= prefix;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) buf[w + __popc(bal & ((1u << lane) - 1u))] = k;
    w += __popc(bal);
    __syncwarp();
  }
  return prefix;
}

// One warp: sort n (<= 512) (block, score) pairs ascending by block in shared memory
// (bitonic network on the next power of two; padding blocks are 0xFFFFFFFF).
__device__ __forceinline__ void warp_sort_blocks(uint32_t* blk, float* sc, int n) {
  const int lane = threadIdx.x & 31;
  int np = 1;
  while (np < n) np <<= 1;
  for (int i = n + lane; i < np; i += 32) {
    blk[i] = 0xFFFFFFFFu;
    sc[i] = 0.f;
  }
  __syncwarp();
  for (int k = 2; k <= np; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < np; i += 32) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint32_t a = blk[i], b = blk[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            blk[i] = b;
            blk[ixj] = a;
            const float t = sc[i];
            sc[i] = sc[ixj];
            sc[ixj] = t;
          }
        }
      }
      __syncwarp();
    }
  }
}

// Row whose query position or sequence failed validation: n_sel = 0, every entry -1.
__device__ __forceinline__ void write_empty_selection(int row, int32_t* sel, int32_t* n_sel,
                                                     float* sel_scores, int stride) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < stride; i += 32) {
    sel[(long long)row * stride + i] = -1;
    if (sel_scores) sel_scores[(long long)row * stride + i] = __int_as_float(0x7fc00000);
  }
  if (lane == 0) n_sel[row] = 0;
}

// Write one row of the selection outputs from n sorted (block, score) pairs plus the tail.
__device__ __forceinline__ void write_selection(int row, int n, int tail, const uint32_t* blk,
                                                const float* sc, int32_t* sel, int32_t* n_sel,
                                                float* sel_scores, int stride) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < stride; i += 32) {
    int32_t b;
    float s;
    if (i < n) {
      b = (int32_t)blk[i];
      s = sc[i];
    } else if (i == n) {
      b = tail;
      s = __int_as_float(0x7f800000);  // +inf marks the tail
    } else {
      b = -1;
      s = __int_as_float(0x7fc00000);  // NaN padding
    }
    sel[(long long)row * stride + i] = b;
    if (sel_scores) sel_scores[(long long)row * stride + i] = s;
  }
  if (lane == 0) n_sel[row] = n + 1;
}

}  // namespace qsa
