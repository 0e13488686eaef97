// Exact top-k selection primitives on 64-bit candidate keys (score major, lower block first).
//
// Keys of one query row are unique (they embed the block index), so "the k largest keys" is a
// well-defined set: the article's selection rule (keep the best 512 micro-blocks) under the
// library's tie-break (lower block index wins).
#pragma once
#include "common.cuh"

namespace qsa {

typedef unsigned long long u64;

// Histogram increment (shared-memory atomic).  Called by all 32 lanes of the warp.
__device__ __forceinline__ void hist_add(uint32_t* h, uint32_t bin, bool active) {
  if (active) atomicAdd(&h[bin], 1u);
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

// One warp: the need-th largest of n unique keys (keys[0..n), shared or global memory), 1 <= need <=
// n.  MSB-first radix select with 11-bit digits that start at the highest bit where the keys
// differ (found from their min and max), so the first pass already spreads them; histogram of
// 2048 words in this warp's shared memory, plain shared atomics.
__device__ __forceinline__ u64 warp_kth_largest2(const u64* ka, int na, const u64* kb, int n, int need,
                                                 uint32_t* hist);
__device__ __forceinline__ u64 warp_kth_largest(const u64* keys, int n, int need, uint32_t* hist) {
  return warp_kth_largest2(keys, n, nullptr, n, need, hist);
}

// Same over the concatenation of two arrays: ka[0..na) then kb[0..n-na).
__device__ __forceinline__ u64 warp_kth_largest2(const u64* ka, int na, const u64* kb, int n, int need,
                                                 uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  auto key_at = [&](int i) { return i < na ? ka[i] : kb[i - na]; };
  u64 lo = ~0ull, hi = 0ull;
  for (int i = lane; i < n; i += 32) {
    const u64 k = key_at(i);
    lo = k < lo ? k : lo;
    hi = k > hi ? k : hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const u64 a = __shfl_xor_sync(0xffffffffu, lo, o), b = __shfl_xor_sync(0xffffffffu, hi, o);
    lo = a < lo ? a : lo;
    hi = b > hi ? b : hi;
  }
  if (need == n) return lo;
  if (need == 1) return hi;
  int top = 63 - __clzll((long long)(lo ^ hi));  // highest differing bit (lo != hi since n >= 2)
  u64 prefix = hi & ~((2ull << top) - 1ull);     // bits above `top` are common to every key
  u64 mask = ~((2ull << top) - 1ull);
  if (top == 63) { prefix = 0; mask = 0; }
  uint32_t remaining = (uint32_t)need;
  for (;;) {
    const int width = top + 1 < 11 ? top + 1 : 11;
    const int shift = top + 1 - width;
    const uint32_t nb = 1u << width;
    for (uint32_t i = lane; i < nb; i += 32) hist[i] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const u64 k = key_at(i);
      if ((k & mask) == prefix) atomicAdd(&hist[(uint32_t)(k >> shift) & (nb - 1)], 1u);
    }
    __syncwarp();
    // lane l owns a contiguous run of bins counted from the top
    const uint32_t per = (nb + 31) / 32;
    uint32_t tot = 0;
    for (uint32_t j = 0; j < per; ++j) {
      const int bin = (int)nb - 1 - (int)(lane * per + j);
      if (bin >= 0) tot += hist[bin];
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
    uint32_t above = 0, cnt_at = 0;
    if (mine) {
      uint32_t acc = excl;
      for (uint32_t j = 0; j < per; ++j) {
        const int bin = (int)nb - 1 - (int)(lane * per + j);
        if (bin < 0) break;
        const uint32_t c = hist[bin];
        if (acc + c >= remaining) {
          digit = bin;
          above = acc;
          cnt_at = c;
          break;
        }
        acc += c;
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    digit = __shfl_sync(0xffffffffu, digit, src);
    above = __shfl_sync(0xffffffffu, above, src);
    cnt_at = __shfl_sync(0xffffffffu, cnt_at, src);
    remaining -= above;
    prefix |= (u64)digit << shift;
    mask |= (u64)(nb - 1) << shift;
    __syncwarp();
    if (shift == 0) return prefix;  // every bit fixed: the key itself
    if (cnt_at == remaining) {      // all keys under this prefix are kept: the answer is their min
      u64 m = ~0ull;
      for (int i = lane; i < n; i += 32) {
        const u64 k = key_at(i);
        if ((k & mask) == prefix && k < m) m = k;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const u64 a = __shfl_xor_sync(0xffffffffu, m, o);
        m = a < m ? a : m;
      }
      return m;
    }
    top = shift - 1;
  }
}

// One warp: keep the keys >= kth of a list that is sorted by block, preserving that order;
// writes blocks and scores to out_blk / out_sc and returns the count.
__device__ __forceinline__ int warp_keep_sorted(const u64* keys, int n, u64 kth, uint32_t* out_blk,
                                                float* out_sc) {
  const int lane = threadIdx.x & 31;
  int w = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const u64 k = i < n ? keys[i] : 0ull;
    const bool keep = i < n && k >= kth;
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int p = w + __popc(bal & ((1u << lane) - 1u));
      out_blk[p] = key_block(k);
      out_sc[p] = key_score(k);
    }
    w += __popc(bal);
  }
  __syncwarp();
  return w;
}

// One warp: write the union of two ascending, disjoint block lists (a: na, b: nb) plus the tail
// as one selection row, placing each element at its rank (own index + elements of the other
// list with a smaller block, by binary search).
__device__ __forceinline__ void warp_write_merged(int row, const uint32_t* ab, const float* as, int na,
                                                  const uint32_t* bb, const float* bs, int nbk,
                                                  int tail, int32_t* sel, int32_t* n_sel,
                                                  float* sel_scores, int stride) {
  const int lane = threadIdx.x & 31;
  int32_t* srow = sel + (long long)row * stride;
  float* crow = sel_scores ? sel_scores + (long long)row * stride : nullptr;
  for (int side = 0; side < 2; ++side) {
    const uint32_t* x = side ? bb : ab;
    const float* xs = side ? bs : as;
    const int nx = side ? nbk : na;
    const uint32_t* y = side ? ab : bb;
    const int ny = side ? na : nbk;
    for (int i = lane; i < nx; i += 32) {
      const uint32_t v = x[i];
      int lo = 0, hi = ny;  // count of y < v
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (y[mid] < v) lo = mid + 1;
        else hi = mid;
      }
      srow[i + lo] = (int32_t)v;
      if (crow) crow[i + lo] = xs[i];
    }
  }
  const int n = na + nbk;
  for (int i = n + lane; i < stride; i += 32) {
    srow[i] = i == n ? tail : -1;
    if (crow) crow[i] = i == n ? __int_as_float(0x7f800000) : __int_as_float(0x7fc00000);
  }
  if (lane == 0) n_sel[row] = n + 1;
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
