/*
 * synth.h -- seeded synthetic inputs for the MoE FFN layer (host and device).
 *
 * This module serves both the oracle and the CUDA layer: it fills the packed
 * weight tensors, the codebook, the router bias and the hash table with
 * counter-based pseudo-random bytes.  It writes fields into the block byte
 * layouts and draws their values; it decodes nothing and performs none of the
 * layer's arithmetic.  The same source is compiled by gcc (host library) and
 * by nvcc (device kernels), so the two fills are byte-identical by
 * construction: every field is produced from integers, and the only floating
 * point (the f16 scales) uses explicitly rounded fp32 multiply and add followed
 * by an integer round-to-nearest-even conversion to binary16.
 *
 * Generator: the SplitMix64 output function of Steele, Lea and Flood
 * ("Fast splittable pseudorandom number generators", OOPSLA 2014), used as a
 * hash of (seed, stream, counter).  A stream is (layer << 8 | tensor id); the
 * counter is the linear block index inside the tensor times 32 plus the word.
 *
 * Distributions (all U = uniform):
 *   IQ2_XXS  d = f16(0.005 + 0.015 u), u = U[0,1) on a 24-bit grid; each
 *            32-element group is one raw 64-bit word, so the four grid
 *            indices are U[0,255], the four 7-bit sign masks U[0,127] and the
 *            4-bit scale U[0,15].
 *   Q2_K     scales/mins bytes and 2-bit codes are raw random bytes (so every
 *            nibble and code is uniform); d, dmin = f16(0.001 + 0.009 u).
 *   Q8_0     d = f16(0.0005); int8 values U[-127,127].
 *   Q4_K     the 12 scale/min bytes and the 4-bit codes are raw random bytes
 *            (every 6-bit scale, 6-bit min and code uniform); d, dmin =
 *            f16(0.0001 + 0.0009 u), so d * 63 * 15 stays below 1.
 *   codebook 256 x 8 bytes, each drawn from {8, 25, 43}.
 *   bias     U(-0.1, 0.1) in fp32, +0.5 on experts with e % 8 == 0 when the
 *            skewed variant is asked for.
 *   tid2eid  per token id, the first k draws of a partial Fisher-Yates
 *            shuffle of 0..n_experts-1 (distinct ids, in draw order).
 */
#ifndef SYNTH_H
#define SYNTH_H

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define SYNTH_FN __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

enum {
  SYNTH_T_BIAS = 2,
  SYNTH_T_GATE = 3,
  SYNTH_T_UP = 4,
  SYNTH_T_DOWN = 5,
  SYNTH_T_SH_GATE = 6,
  SYNTH_T_SH_UP = 7,
  SYNTH_T_SH_DOWN = 8,
  SYNTH_T_GRID = 9,
  SYNTH_T_TID2EID = 10,
};

enum { SYNTH_IQ2XXS_BYTES = 66, SYNTH_Q2K_BYTES = 84, SYNTH_Q80_BYTES = 34, SYNTH_Q4K_BYTES = 144 };

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

SYNTH_FN uint64_t synth_key(uint64_t seed, uint32_t layer, uint32_t tensor) {
  return synth_mix64(synth_mix64(seed) ^ (((uint64_t)layer << 8) | tensor));
}

SYNTH_FN uint64_t synth_word(uint64_t key, uint64_t block, uint32_t word) {
  return synth_mix64(key ^ synth_mix64((block << 5) | word));
}

/* uniform integer in [0, n) from the high 32 bits (multiply-shift). */
SYNTH_FN uint32_t synth_below(uint64_t v, uint32_t n) {
  return (uint32_t)(((v >> 32) * (uint64_t)n) >> 32);
}

SYNTH_FN uint32_t synth_f32_bits(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
#endif
}

/* lo + (hi - lo) * (u24 / 2^24) with each fp32 operation rounded on its own. */
SYNTH_FN float synth_affine24(uint32_t u24, float lo, float span) {
  float u = (float)u24 * (1.0f / 16777216.0f); /* exact */
#if defined(__CUDA_ARCH__)
  return __fadd_rn(lo, __fmul_rn(span, u));
#else
  volatile float p = span * u;
  return lo + p;
#endif
}

/* fp32 -> IEEE binary16, round to nearest even, integer arithmetic only. */
SYNTH_FN uint16_t synth_f16_bits(float f) {
  uint32_t x = synth_f32_bits(f);
  uint32_t sign = (x >> 16) & 0x8000u;
  uint32_t ax = x & 0x7FFFFFFFu;
  if (ax >= 0x7F800000u) return (uint16_t)(sign | 0x7C00u | (ax > 0x7F800000u ? 0x200u : 0u));
  if (ax >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u); /* rounds past 65504 */
  if (ax < 0x38800000u) {                                     /* f16 subnormal or zero */
    if (ax < 0x33000000u) return (uint16_t)sign;               /* below half the least subnormal */
    uint32_t e = ax >> 23;
    uint32_t m = (ax & 0x7FFFFFu) | 0x800000u;
    uint32_t shift = 126u - e; /* value = m * 2^(e-150); subnormal unit 2^-24 */
    uint32_t q = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1u);
    if (rem > half || (rem == half && (q & 1u))) q++;
    return (uint16_t)(sign | q);
  }
  uint32_t e = (ax >> 23) - 112u; /* rebias 127 -> 15 */
  uint32_t m = ax & 0x7FFFFFu;
  uint32_t q = (e << 10) | (m >> 13);
  uint32_t rem = m & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (q & 1u))) q++;
  return (uint16_t)(sign | q);
}

SYNTH_FN void synth_put16(uint8_t *p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xFF);
  p[1] = (uint8_t)(v >> 8);
}

SYNTH_FN void synth_put64(uint8_t *p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}

/* One IQ2_XXS block (256 elements, 66 bytes): f16 d, then 8 groups of 8 bytes. */
SYNTH_FN void synth_iq2xxs_block(uint64_t key, uint64_t block, uint8_t *out) {
  uint64_t w0 = synth_word(key, block, 0);
  synth_put16(out, synth_f16_bits(synth_affine24((uint32_t)(w0 >> 40), 0.005f, 0.015f)));
  for (int g = 0; g < 8; ++g) synth_put64(out + 2 + 8 * g, synth_word(key, block, 1 + g));
}

/* One Q2_K block (256 elements, 84 bytes): scales[16], qs[64], f16 d, f16 dmin. */
SYNTH_FN void synth_q2k_block(uint64_t key, uint64_t block, uint8_t *out) {
  for (int w = 0; w < 10; ++w) synth_put64(out + 8 * w, synth_word(key, block, w));
  uint64_t wd = synth_word(key, block, 10);
  synth_put16(out + 80, synth_f16_bits(synth_affine24((uint32_t)(wd >> 40), 0.001f, 0.009f)));
  synth_put16(out + 82, synth_f16_bits(synth_affine24((uint32_t)(wd >> 8) & 0xFFFFFFu, 0.001f, 0.009f)));
}

/* One Q8_0 block (32 elements, 34 bytes): f16 d, int8 q[32] in [-127, 127]. */
SYNTH_FN void synth_q80_block(uint64_t key, uint64_t block, uint8_t *out) {
  synth_put16(out, synth_f16_bits(0.0005f));
  for (int w = 0; w < 16; ++w) {
    uint64_t v = synth_word(key, block, w);
    int32_t a = (int32_t)synth_below(v, 255u) - 127;
    int32_t b = (int32_t)synth_below(v << 32, 255u) - 127;
    out[2 + 2 * w] = (uint8_t)(int8_t)a;
    out[3 + 2 * w] = (uint8_t)(int8_t)b;
  }
}

/* One Q4_K block (256 elements, 144 bytes): f16 d, f16 dmin, then 140 raw
 * bytes (12 of scales and mins, 128 of codes). */
SYNTH_FN void synth_q4k_block(uint64_t key, uint64_t block, uint8_t *out) {
  for (int w = 0; w < 17; ++w) synth_put64(out + 4 + 8 * w, synth_word(key, block, w)); /* bytes 4..139 */
  uint64_t wt = synth_word(key, block, 17);
  for (int i = 0; i < 4; ++i) out[140 + i] = (uint8_t)(wt >> (8 * i));
  uint64_t wd = synth_word(key, block, 18);
  synth_put16(out, synth_f16_bits(synth_affine24((uint32_t)(wd >> 40), 0.0001f, 0.0009f)));
  synth_put16(out + 2, synth_f16_bits(synth_affine24((uint32_t)(wd >> 8) & 0xFFFFFFu, 0.0001f, 0.0009f)));
}

/* Codebook entry (row r, lane l) drawn from {8, 25, 43}. */
SYNTH_FN uint8_t synth_grid_entry(uint64_t key, uint32_t r, uint32_t l) {
  const uint8_t vals[3] = {8, 25, 43};
  return vals[synth_below(synth_word(key, r, l), 3u)];
}

SYNTH_FN float synth_bias(uint64_t key, uint32_t e, int skew) {
  float b = synth_affine24((uint32_t)(synth_word(key, e, 0) >> 40), -0.1f, 0.2f);
  if (skew && (e % 8u) == 0u) {
#if defined(__CUDA_ARCH__)
    b = __fadd_rn(b, 0.5f);
#else
    volatile float t = b + 0.5f;
    b = t;
#endif
  }
  return b;
}

/* k distinct expert ids for one token id: partial Fisher-Yates over 0..E-1. */
SYNTH_FN void synth_tid2eid_row(uint64_t key, uint32_t tid, int n_experts, int k, int32_t *out) {
  int32_t perm[256];
  for (int i = 0; i < n_experts; ++i) perm[i] = i;
  for (int i = 0; i < k; ++i) {
    uint32_t j = (uint32_t)i + synth_below(synth_word(key, tid, (uint32_t)i), (uint32_t)(n_experts - i));
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
    out[i] = perm[i];
  }
}

#endif /* SYNTH_H */
