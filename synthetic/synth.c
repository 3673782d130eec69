/*
 * Host implementation of the seeded input generator (definition in synth.h).
 * Compiled with -ffp-contract=off so that every fp operation is rounded on its
 * own, exactly as the device implementation does with __fmul_rn/__dadd_rn.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "synth.h"

static inline uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

static inline uint16_t f32_to_f16_bits(float f) {
  _Float16 h = (_Float16)f; /* IEEE round-to-nearest-even */
  uint16_t u;
  memcpy(&u, &h, 2);
  return u;
}

static inline float std_normal(uint64_t key, uint64_t i) {
  return (float)synth_irwin_hall12(key, i) * (1.0f / 65536.0f);
}

/* out[j] = N(0, sigma^2) draw number offset+j of tensor (seed, tensor_id). */
void synth_host_normal(uint64_t seed, uint64_t tensor_id, uint64_t offset, uint64_t n,
                       float sigma, int dtype, void* out) {
  const uint64_t key = synth_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)n; ++j) {
    float v = std_normal(key, offset + (uint64_t)j) * sigma;
    if (dtype == SYNTH_DT_F32) {
      ((float*)out)[j] = v;
    } else if (dtype == SYNTH_DT_BF16) {
      ((uint16_t*)out)[j] = synth_f32_to_bf16_bits(f32_bits(v));
    } else {
      ((uint16_t*)out)[j] = f32_to_f16_bits(v);
    }
  }
}

/* Rows row0..row0+rows-1 of a [*, cols] matrix: g ~ N(0,1), then each row is
 * divided by sqrt(mean(g^2) + 1e-6) in double (sequential sum in column
 * order), converted to fp32 and rounded to the storage type. */
void synth_host_rmsnorm_rows(uint64_t seed, uint64_t tensor_id, int64_t row0, int64_t rows,
                             int64_t cols, int dtype, void* out) {
  const uint64_t key = synth_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)cols;
    double ss = 0.0;
    for (int64_t c = 0; c < cols; ++c) {
      double g = (double)std_normal(key, base + (uint64_t)c);
      ss = ss + g * g;
    }
    double rms = sqrt(ss / (double)cols + 1e-6);
    for (int64_t c = 0; c < cols; ++c) {
      double g = (double)std_normal(key, base + (uint64_t)c);
      float v = (float)(g / rms);
      int64_t o = r * cols + c;
      if (dtype == SYNTH_DT_F32) {
        ((float*)out)[o] = v;
      } else if (dtype == SYNTH_DT_BF16) {
        ((uint16_t*)out)[o] = synth_f32_to_bf16_bits(f32_bits(v));
      } else {
        ((uint16_t*)out)[o] = f32_to_f16_bits(v);
      }
    }
  }
}

/* q4_0 matrix rows row0..row0+rows-1 of a [*, cols] matrix (cols % 32 == 0):
 * qs[r][cols/2] random nibble bytes, scales[r][cols/32] fp16 codes. */
void synth_host_q4(uint64_t seed, uint64_t tensor_id, int64_t row0, int64_t rows, int64_t cols,
                   uint8_t* qs, uint16_t* scales) {
  const uint64_t key = synth_key(seed, tensor_id);
  const int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      uint64_t gi = (uint64_t)((row0 + r) * nb + b);
      scales[r * nb + b] = synth_q4_scale_code(key, gi);
      for (int j = 0; j < 16; ++j) qs[r * (cols / 2) + b * 16 + j] = synth_q4_byte(key, gi, j);
    }
  }
}
