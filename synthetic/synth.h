/*
 * Seeded synthetic inputs for the MoE layer forward.
 *
 * This module is input preparation only: it draws the activations and weights
 * that both the CPU oracle and the GPU path consume.  It contains none of the
 * layer's arithmetic (no router, softmax, top-k, permutation, SwiGLU or
 * combine).  The host implementation (synth.c) and the device implementation
 * (synth_cuda.cu) produce bit-identical values: every draw is integer hashing
 * plus exactly rounded IEEE operations that both sides evaluate in the same
 * order without contraction.
 *
 * Generator definition (counter based, no state):
 *   splitmix64(x): Vigna's published mixer (golden-gamma increment, then two
 *                  xor-shift-multiply rounds and a final xor-shift).
 *   key(seed, tensor_id) = splitmix64(seed * 0x9E3779B97F4A7C15 ^ splitmix64(tensor_id))
 *   standard normal #i:  s = sum of the twelve 16-bit fields of
 *                        splitmix64(key + 3i + j), j = 0, 1, 2
 *                        x = float(s - 393210) * 2^-16   (exact; Irwin-Hall n=12)
 *   scaled:              v = x * sigma                  (one fp32 multiply, RN)
 *   bf16 / fp16:         round-to-nearest-even of the fp32 value.
 */
#ifndef MOE_SYNTH_H
#define MOE_SYNTH_H

#include <stdint.h>

#ifdef __CUDACC__
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

#define SYNTH_DT_F32 0
#define SYNTH_DT_BF16 1
#define SYNTH_DT_F16 2

SYNTH_HD uint64_t synth_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

SYNTH_HD uint64_t synth_key(uint64_t seed, uint64_t tensor_id) {
  return synth_splitmix64((seed * 0x9E3779B97F4A7C15ull) ^ synth_splitmix64(tensor_id));
}

/* Sum of twelve 16-bit uniforms minus their mean, as an exact integer. */
SYNTH_HD int64_t synth_irwin_hall12(uint64_t key, uint64_t i) {
  int64_t s = 0;
  for (int j = 0; j < 3; ++j) {
    uint64_t h = synth_splitmix64(key + 3ull * i + (uint64_t)j);
    s += (int64_t)(h & 0xFFFFull) + (int64_t)((h >> 16) & 0xFFFFull) +
         (int64_t)((h >> 32) & 0xFFFFull) + (int64_t)(h >> 48);
  }
  return s - 393210;
}

/* fp32 -> bf16 round-to-nearest-even on the bit pattern (finite inputs). */
SYNTH_HD uint16_t synth_f32_to_bf16_bits(uint32_t u) {
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* q4_0 block scale code (fp16 bit pattern) for global block index gi.
 * One block in 64 gets a zero scale, 7 in 64 a subnormal scale, the rest a
 * normal scale in [2^-9, 2^-7) with a random sign. */
SYNTH_HD uint16_t synth_q4_scale_code(uint64_t key, uint64_t gi) {
  uint64_t h = synth_splitmix64(key ^ 0x5CA1E5ull) ;
  h = synth_splitmix64(h + gi);
  uint16_t sign = (uint16_t)(((h >> 30) & 1ull) << 15);
  if ((h & 63ull) == 0ull) return 0;
  if ((h & 7ull) == 0ull) return (uint16_t)(sign | (uint16_t)(1u + (uint32_t)((h >> 8) % 1023ull)));
  uint16_t ex = (uint16_t)(6u + (uint32_t)((h >> 20) & 1ull));
  uint16_t man = (uint16_t)((h >> 40) & 0x3FFull);
  return (uint16_t)(sign | (uint16_t)(ex << 10) | man);
}

/* Byte b (0..15) of q4_0 block gi: two random nibbles. */
SYNTH_HD uint8_t synth_q4_byte(uint64_t key, uint64_t gi, int b) {
  uint64_t h = synth_splitmix64(key + 2ull * gi + (uint64_t)(b >> 3));
  return (uint8_t)((h >> (8 * (b & 7))) & 0xFFull);
}

#endif
