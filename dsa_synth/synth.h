/*
 * synth.h - counter-based synthetic input generator for the gated
 * Indexer + Top-K sparse-attention layer.
 *
 * This module makes the seeded inputs that both the CPU oracle and the CUDA
 * path consume.  It holds none of the layer's arithmetic: it only turns
 * (seed, tensor id, flat element index) into a value, identically on the host
 * and on the device, using integer operations and one correctly rounded fp32
 * multiply.  No transcendental function is used, so host and device agree
 * bit for bit.
 *
 * Value families (all drawn per element, independent of launch shape):
 *   grid    : (h mod 9 - 4) / 8, the "dyadic grid" {-4..4}/8.  Exact in bf16
 *             and in fp8 e4m3, so indexer dot products are exact in fp32.
 *   normal  : Irwin-Hall sum of twelve 16-bit uniforms minus 6 (mean 0,
 *             variance 1), times an fp32 scale, rounded to bf16 (RNE).
 *   weight  : {0.25, 0.5, 1}[h mod 3], an fp32 indexer head weight.
 *
 * Hash: splitmix64's finaliser (Steele, Lea, Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) applied twice.
 */
#ifndef DSA_SYNTH_H
#define DSA_SYNTH_H

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* tensor ids: every input tensor of a workload draws from its own stream */
enum {
  SYNTH_T_Q_IDX = 1,
  SYNTH_T_K_IDX = 2,
  SYNTH_T_W = 3,
  SYNTH_T_Q = 4,
  SYNTH_T_K = 5,
  SYNTH_T_V = 6,
  SYNTH_T_GATE = 7,
  SYNTH_T_SCORES = 8,
  SYNTH_T_LAYOUT = 9,  /* ragged lengths, needle positions, signs */
};

/* value families */
enum {
  SYNTH_GRID = 0,
  SYNTH_NORMAL = 1,
  SYNTH_WEIGHT = 2,
  SYNTH_ZERO = 3,
  SYNTH_ONE = 4,
};

SYNTH_HD uint64_t synth_mix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

SYNTH_HD uint64_t synth_hash(uint64_t seed, uint32_t tensor, uint64_t i) {
  uint64_t stream = synth_mix64(seed ^ ((uint64_t)tensor * 0xD1B54A32D192ED03ull));
  return synth_mix64(stream ^ i);
}

SYNTH_HD float synth_bits_f32(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

SYNTH_HD uint32_t synth_f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* fp32 -> bf16 bit pattern, round to nearest even (finite inputs). */
SYNTH_HD uint16_t synth_f32_to_bf16(float f) {
  uint32_t u = synth_f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

SYNTH_HD float synth_bf16_to_f32(uint16_t b) { return synth_bits_f32((uint32_t)b << 16); }

/* grid value index k in [0, 9): value (k - 4) / 8 */
SYNTH_HD int synth_grid_code(uint64_t h) { return (int)(h % 9u); }

SYNTH_HD float synth_grid_value(uint64_t h) { return (float)(synth_grid_code(h) - 4) * 0.125f; }

/* e4m3 (bias 7) bit patterns of (k - 4) / 8 for k = 0..8 */
SYNTH_HD uint8_t synth_grid_e4m3(uint64_t h) {
  /* |v| = 0.5 -> 0x30, 0.375 -> 0x2C, 0.25 -> 0x28, 0.125 -> 0x20, 0 -> 0x00 */
  int k = synth_grid_code(h) - 4;
  int a = k < 0 ? -k : k;
  uint8_t mag = a == 4 ? 0x30 : a == 3 ? 0x2C : a == 2 ? 0x28 : a == 1 ? 0x20 : 0x00;
  return (uint8_t)(k < 0 ? (mag | 0x80) : mag);
}

/* Irwin-Hall(12) - 6 as an exact fp32 value, then times scale (one RNE multiply). */
SYNTH_HD float synth_normal(uint64_t seed, uint32_t tensor, uint64_t i, float scale) {
  uint32_t s = 0;
  for (int r = 0; r < 3; ++r) {
    uint64_t h = synth_hash(seed, tensor, 3ull * i + (uint64_t)r);
    s += (uint32_t)(h & 0xFFFFu) + (uint32_t)((h >> 16) & 0xFFFFu) +
         (uint32_t)((h >> 32) & 0xFFFFu) + (uint32_t)((h >> 48) & 0xFFFFu);
  }
  float x = (float)((int32_t)s - 6 * 65536) * (1.0f / 65536.0f); /* exact */
#if defined(__CUDA_ARCH__)
  return __fmul_rn(x, scale);
#else
  volatile float xs = x * scale;
  return xs;
#endif
}

SYNTH_HD float synth_weight(uint64_t h) {
  uint32_t k = (uint32_t)(h % 3u);
  return k == 0 ? 0.25f : (k == 1 ? 0.5f : 1.0f);
}

/* One bf16 element (as bits) of the given family. */
SYNTH_HD uint16_t synth_bf16_elem(int family, uint64_t seed, uint32_t tensor, uint64_t i,
                                  float scale) {
  switch (family) {
    case SYNTH_GRID:
      return synth_f32_to_bf16(synth_grid_value(synth_hash(seed, tensor, i)));
    case SYNTH_NORMAL:
      return synth_f32_to_bf16(synth_normal(seed, tensor, i, scale));
    case SYNTH_ONE:
      return synth_f32_to_bf16(scale);
    default:
      return 0;
  }
}

#ifdef __cplusplus
}
#endif

#endif /* DSA_SYNTH_H */
