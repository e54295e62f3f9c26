/*
 * synth_core.h -- counter-based seeded input generator, shared by the host
 * (C, synth.c) and device (CUDA, synth_dev.cu) builds of the generator.
 *
 * This file holds no arithmetic of the MoE method.  It only turns a
 * (seed, layer, expert, tensor, element) key into pseudo-random bits and
 * maps bits to the input distributions of the synthetic workloads:
 *   - packed int4 weight bytes: raw random bytes (each nibble is then uniform
 *     over the 16 two's-complement codes -8..7);
 *   - fp16 scales: U(lo, hi) computed in double, rounded to fp16 (RNE);
 *   - fp32 / bf16 values from N(0, sigma) or U(lo, hi) (host only, libm).
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Element i of a stream with
 * key K is the i-th output of SplitMix64 seeded with K:
 *     draw(K, i) = mix64(K + (i + 1) * GAMMA)
 * mix64 is SplitMix64's output finaliser.  Everything here is integer or
 * explicitly rounded double arithmetic, so the host and device builds give
 * identical bits.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

/* Tensor tags: the fourth component of a stream key. */
enum {
  SYNTH_T_Q_GATE = 0,
  SYNTH_T_Q_UP = 1,
  SYNTH_T_Q_DOWN = 2,
  SYNTH_T_S_GATE = 3,
  SYNTH_T_S_UP = 4,
  SYNTH_T_S_DOWN = 5,
  SYNTH_T_W_ROUTER = 6,
  SYNTH_T_BIAS = 7,
  SYNTH_T_X = 8,        /* expert field = token stream index */
  SYNTH_T_EPS = 9,      /* perturbation of the correlated batch variant */
  SYNTH_T_PERM = 10,    /* per-layer expert permutation of the Zipf trace */
  SYNTH_T_TRACE = 11    /* per-token draws of the Zipf trace */
};

SYNTH_HD uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Stream key for (seed, layer, expert, tensor). */
SYNTH_HD uint64_t synth_key(uint64_t seed, uint32_t layer, uint32_t expert,
                            uint32_t tensor) {
  uint64_t k = synth_mix64(seed + SYNTH_GAMMA);
  k = synth_mix64(k ^ ((uint64_t)layer + 1) * SYNTH_GAMMA);
  k = synth_mix64(k ^ ((uint64_t)expert + 1) * 0xD1B54A32D192ED03ULL);
  k = synth_mix64(k ^ ((uint64_t)tensor + 1) * 0x8CB92BA72F3D8DD7ULL);
  return k;
}

SYNTH_HD uint64_t synth_draw(uint64_t key, uint64_t i) {
  return synth_mix64(key + (i + 1) * SYNTH_GAMMA);
}

/* Uniform double in [0, 1) with 53 random bits. */
SYNTH_HD double synth_u53(uint64_t r) {
  return (double)(r >> 11) * (1.0 / 9007199254740992.0);
}

/* Round a finite double to IEEE binary16, round-to-nearest-even, using only
 * integer operations on the bit pattern.  Overflow saturates to +-inf. */
SYNTH_HD uint16_t synth_f64_to_f16(double d) {
  union { double d; uint64_t u; } v;
  v.d = d;
  uint64_t u = v.u;
  uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  int e = (int)((u >> 52) & 0x7FF);
  uint64_t m = u & 0xFFFFFFFFFFFFFULL;
  if (e == 0x7FF) return (uint16_t)(sign | 0x7C00u | (m ? 0x200u : 0u));
  int ue = e - 1023;                       /* unbiased exponent */
  if (e == 0 || ue < -25) return sign;     /* |d| < 2^-25 rounds to zero */
  uint64_t sig = m | (1ULL << 52);         /* 53-bit significand */
  if (ue >= -14) {                         /* normal fp16 (before rounding) */
    /* keep 11 bits: shift right by 42 */
    uint64_t keep = sig >> 42;
    uint64_t rem = sig & ((1ULL << 42) - 1);
    uint64_t half = 1ULL << 41;
    if (rem > half || (rem == half && (keep & 1))) keep++;
    int he = ue + 15;
    if (keep == (1ULL << 11)) { keep >>= 1; he++; }
    if (he >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | ((uint16_t)he << 10) | (uint16_t)(keep & 0x3FF));
  }
  /* subnormal fp16: value = sig * 2^(ue-52); unit is 2^-24 */
  int shift = 42 + (-14 - ue);             /* 43..53 */
  uint64_t keep = sig >> shift;
  uint64_t rem = sig & ((1ULL << shift) - 1);
  uint64_t half = 1ULL << (shift - 1);
  if (rem > half || (rem == half && (keep & 1))) keep++;
  return (uint16_t)(sign | (uint16_t)keep);  /* keep==1024 gives min normal */
}

/* Round a float to bfloat16, round-to-nearest-even (finite inputs). */
SYNTH_HD uint16_t synth_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Byte b of a packed-int4 stream: byte (b & 7) of draw b >> 3, little-endian. */
SYNTH_HD uint8_t synth_byte(uint64_t key, uint64_t b) {
  return (uint8_t)(synth_draw(key, b >> 3) >> (8 * (b & 7)));
}

/* Explicitly rounded double ops, so no build fuses a multiply-add. */
#if defined(__CUDA_ARCH__)
#define SYNTH_DMUL(a, b) __dmul_rn((a), (b))
#define SYNTH_DADD(a, b) __dadd_rn((a), (b))
#else
#define SYNTH_DMUL(a, b) ((a) * (b))
#define SYNTH_DADD(a, b) ((a) + (b))
#endif

/* Element i of an fp16 scale stream: U(lo, hi) in double, rounded to fp16. */
SYNTH_HD uint16_t synth_scale_f16(uint64_t key, uint64_t i, double lo,
                                  double hi) {
  double u = synth_u53(synth_draw(key, i));
  return synth_f64_to_f16(SYNTH_DADD(lo, SYNTH_DMUL(hi - lo, u)));
}

#endif /* SYNTH_CORE_H */
