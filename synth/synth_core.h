/* Counter-based synthetic tensor generator: the element functions.
 *
 * Every synthetic input of the MoE layer (hidden states, router centroids,
 * expert weights, selection bias) is a pure function of (key, index), where
 * key = syn_key(seed, tensor_id) and index is the element's row-major flat
 * index.  Any element, or any block of a tensor (one expert's weights), can
 * therefore be regenerated on its own, on the host or on the device, with
 * bit-identical results.  Only integer operations and single correctly
 * rounded IEEE operations are used, so host and device agree exactly.
 *
 * This header holds input generation only: nothing of the MoE method's
 * arithmetic lives here.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_FN __host__ __device__ __forceinline__
#else
#define SYN_FN static inline
#endif

/* splitmix64: Weyl sequence with increment 0x9E3779B97F4A7C15 followed by the
 * finaliser of Steele, Lea and Flood ("Fast splittable pseudorandom number
 * generators", OOPSLA 2014). */
#define SYN_GAMMA 0x9E3779B97F4A7C15ull

SYN_FN uint64_t syn_mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

/* Per-tensor key: two splitmix64 outputs chained over (seed, tensor_id). */
SYN_FN uint64_t syn_key(uint64_t seed, uint64_t tensor_id) {
  return syn_mix64(syn_mix64(seed + SYN_GAMMA) + (tensor_id + 1) * SYN_GAMMA);
}

/* Element `index` of the stream with key `key`: splitmix64 state at
 * position index+1 of the Weyl sequence started at key. */
SYN_FN uint64_t syn_bits(uint64_t key, uint64_t index) {
  return syn_mix64(key + (index + 1) * SYN_GAMMA);
}

/* Approximate standard normal, unscaled: Irwin-Hall sum of four independent
 * 16-bit uniform integers, centred.  The result is an integer in
 * [-131070, 131070] with mean 0 and variance (65536^2 - 1) / 3; it is exact in
 * fp32 (|value| < 2^24). */
SYN_FN int32_t syn_irwin_hall4(uint64_t h) {
  int32_t a = (int32_t)(h & 0xFFFFu);
  int32_t b = (int32_t)((h >> 16) & 0xFFFFu);
  int32_t c = (int32_t)((h >> 32) & 0xFFFFu);
  int32_t d = (int32_t)((h >> 48) & 0xFFFFu);
  return a + b + c + d - 131070;
}

/* Normal-like value: one correctly rounded fp32 multiply of an exact integer
 * by `scale` (= sigma / sqrt((65536^2 - 1) / 3), rounded to fp32 by the
 * caller). */
#if defined(__CUDA_ARCH__)
#define SYN_FMUL(a, b) __fmul_rn((a), (b))
#define SYN_DMUL(a, b) __dmul_rn((a), (b))
#define SYN_DADD(a, b) __dadd_rn((a), (b))
#else
#define SYN_FMUL(a, b) ((a) * (b))
#define SYN_DMUL(a, b) ((a) * (b))
#define SYN_DADD(a, b) ((a) + (b))
#endif

SYN_FN float syn_normal_f32(uint64_t key, uint64_t index, float scale) {
  return SYN_FMUL((float)syn_irwin_hall4(syn_bits(key, index)), scale);
}

/* Uniform on [lo, hi): 24-bit uniform u in [0,1), then lo + (hi-lo)*u in
 * fp64 with two separately rounded operations, then one rounding to fp32. */
SYN_FN float syn_uniform_f32(uint64_t key, uint64_t index, float lo, float hi) {
  double u = (double)(syn_bits(key, index) >> 40) * (1.0 / 16777216.0);
  double w = (double)hi - (double)lo;
  return (float)SYN_DADD((double)lo, SYN_DMUL(w, u));
}

/* fp32 -> bf16 bit pattern, round to nearest even (finite inputs). */
SYN_FN uint16_t syn_f32_to_bf16_bits(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t r = v.u + 0x7FFFu + ((v.u >> 16) & 1u);
  return (uint16_t)(r >> 16);
}

#endif /* SYNTH_CORE_H */
