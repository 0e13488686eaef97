/*
 * qsa_synth/gen_core.h -- the counter-based input generator, device/host side.
 *
 * This module makes the seeded synthetic inputs (queries, keys, values, head
 * weights) that both the CUDA path and the CPU oracle consume.  It holds none
 * of the attention method's arithmetic.  The numpy twin in
 * qsa_synth/__init__.py computes the same bits on the host; a GPU test checks
 * the two agree element for element.
 *
 * Generator: element i of tensor `tid` under seed `seed` is the (i+1)-th
 * output of a SplitMix64 stream (Steele, Lea & Flood, "Fast Splittable
 * Pseudorandom Number Generators", OOPSLA 2014; finaliser constants as in
 * Vigna's public-domain splitmix64.c) whose starting state is itself the first
 * SplitMix64 output of state (seed << 20) ^ tid.
 *
 * Distributions (all end in a bf16 bit pattern, rounded to nearest-even with
 * integer operations so that host and device agree bit for bit):
 *   QSYN_NORMAL   Irwin-Hall stand-in for N(0,1): the sum of the four 16-bit
 *                 lanes of the hash, centred (integer), times fp32(sqrt 3),
 *                 times 2^-16.  Mean 0, variance 1, bounded by +-3.46.
 *   QSYN_UNIFORM  U[0,1): top 24 bits of the hash times 2^-24 (exact).
 *   QSYN_INT3     integers -3..3: ((hash >> 32) mod 7) - 3 (exact in bf16).
 */
#ifndef QSA_SYNTH_GEN_CORE_H
#define QSA_SYNTH_GEN_CORE_H
#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define QSYN_HD __host__ __device__ __forceinline__
#else
#define QSYN_HD static inline
#endif

enum { QSYN_NORMAL = 0, QSYN_UNIFORM = 1, QSYN_INT3 = 2 };

#define QSYN_GAMMA 0x9E3779B97F4A7C15ULL

QSYN_HD uint64_t qsyn_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Starting state of the stream for (seed, tid). */
QSYN_HD uint64_t qsyn_key(uint64_t seed, uint64_t tid) {
  return qsyn_mix(((seed << 20) ^ tid) + QSYN_GAMMA);
}

/* Hash of element i: the (i+1)-th output of the stream. */
QSYN_HD uint64_t qsyn_hash(uint64_t key, uint64_t i) {
  return qsyn_mix(key + (i + 1ULL) * QSYN_GAMMA);
}

/* fp32 bits -> bf16 bits, round to nearest even (inputs here are finite). */
QSYN_HD uint16_t qsyn_f32bits_to_bf16(uint32_t u) {
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

#ifdef __CUDACC__
QSYN_HD uint32_t qsyn_f2u(float f) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(f);
#else
  uint32_t u; memcpy(&u, &f, 4); return u;
#endif
}
QSYN_HD float qsyn_mul_rn(float a, float b) {
#ifdef __CUDA_ARCH__
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}
#endif

/* bf16 bit pattern of element with hash h under distribution dist. */
#ifdef __CUDACC__
QSYN_HD uint16_t qsyn_value_bf16(uint64_t h, int dist) {
  if (dist == QSYN_NORMAL) {
    int32_t s = (int32_t)(h & 0xFFFF) + (int32_t)((h >> 16) & 0xFFFF) +
                (int32_t)((h >> 32) & 0xFFFF) + (int32_t)((h >> 48) & 0xFFFF);
    float f = qsyn_mul_rn((float)(s - 131070), 1.7320508075688772f);
    f = qsyn_mul_rn(f, 1.52587890625e-05f); /* 2^-16, exact */
    return qsyn_f32bits_to_bf16(qsyn_f2u(f));
  } else if (dist == QSYN_UNIFORM) {
    float f = qsyn_mul_rn((float)(uint32_t)(h >> 40), 5.9604644775390625e-08f); /* 2^-24 */
    return qsyn_f32bits_to_bf16(qsyn_f2u(f));
  } else {
    int32_t v = (int32_t)((h >> 32) % 7ULL) - 3;
    return qsyn_f32bits_to_bf16(qsyn_f2u((float)v));
  }
}
#endif

#endif
