// Device implementation of the seeded input generator (definition in synth.h).
// Every floating-point step uses an explicitly rounded intrinsic so that no
// fused multiply-add can change a value relative to the host implementation.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth.h"

namespace {

__device__ __forceinline__ float std_normal(uint64_t key, uint64_t i) {
  return __fmul_rn((float)synth_irwin_hall12(key, i), 1.0f / 65536.0f);
}

__device__ __forceinline__ void store(void* out, int dtype, uint64_t o, float v) {
  if (dtype == SYNTH_DT_F32) {
    ((float*)out)[o] = v;
  } else if (dtype == SYNTH_DT_BF16) {
    ((__nv_bfloat16*)out)[o] = __float2bfloat16_rn(v);
  } else {
    ((__half*)out)[o] = __float2half_rn(v);
  }
}

__global__ void normal_kernel(uint64_t key, uint64_t offset, uint64_t n, float sigma, int dtype,
                              void* out) {
  for (uint64_t j = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; j < n;
       j += (uint64_t)gridDim.x * blockDim.x) {
    store(out, dtype, j, __fmul_rn(std_normal(key, offset + j), sigma));
  }
}

// One warp per row; the sum of squares is sequential in column order (lane 0
// accumulates) to match the host definition exactly.
__global__ void rmsnorm_rows_kernel(uint64_t key, int64_t row0, int64_t rows, int64_t cols,
                                    int dtype, void* out) {
  int64_t r = blockIdx.x * (int64_t)(blockDim.x / 32) + threadIdx.x / 32;
  int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)cols;
  double rms = 0.0;
  if (lane == 0) {
    double ss = 0.0;
    for (int64_t c = 0; c < cols; ++c) {
      double g = (double)std_normal(key, base + (uint64_t)c);
      ss = __dadd_rn(ss, __dmul_rn(g, g));
    }
    rms = __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)cols), 1e-6));
  }
  rms = __shfl_sync(0xffffffffu, rms, 0);
  for (int64_t c = lane; c < cols; c += 32) {
    double g = (double)std_normal(key, base + (uint64_t)c);
    store(out, dtype, (uint64_t)(r * cols + c), __double2float_rn(__ddiv_rn(g, rms)));
  }
}

__global__ void q4_kernel(uint64_t key, int64_t row0, int64_t rows, int64_t cols, uint8_t* qs,
                          uint16_t* scales) {
  const int64_t nb = cols / 32;
  const int64_t total = rows * nb;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    int64_t r = t / nb, b = t % nb;
    uint64_t gi = (uint64_t)((row0 + r) * nb + b);
    scales[t] = synth_q4_scale_code(key, gi);
    uint8_t* q = qs + r * (cols / 2) + b * 16;
    for (int j = 0; j < 16; ++j) q[j] = synth_q4_byte(key, gi, j);
  }
}

int grid_for(uint64_t n) {
  uint64_t g = (n + 255) / 256;
  if (g > 148ull * 64ull) g = 148ull * 64ull;
  if (g == 0) g = 1;
  return (int)g;
}

}  // namespace

extern "C" int synth_dev_normal(uint64_t seed, uint64_t tensor_id, uint64_t offset, uint64_t n,
                                float sigma, int dtype, void* out, void* stream) {
  if (n == 0) return 0;
  if (!out || dtype < 0 || dtype > 2) return -1;
  normal_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(synth_key(seed, tensor_id), offset,
                                                               n, sigma, dtype, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

extern "C" int synth_dev_rmsnorm_rows(uint64_t seed, uint64_t tensor_id, int64_t row0,
                                      int64_t rows, int64_t cols, int dtype, void* out,
                                      void* stream) {
  if (rows == 0) return 0;
  if (!out || dtype < 0 || dtype > 2 || cols <= 0) return -1;
  int blocks = (int)((rows + 7) / 8);
  rmsnorm_rows_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(synth_key(seed, tensor_id), row0,
                                                                rows, cols, dtype, out);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

extern "C" int synth_dev_q4(uint64_t seed, uint64_t tensor_id, int64_t row0, int64_t rows,
                            int64_t cols, uint8_t* qs, uint16_t* scales, void* stream) {
  if (rows == 0) return 0;
  if (!qs || !scales || cols % 32 != 0) return -1;
  q4_kernel<<<grid_for((uint64_t)(rows * (cols / 32))), 256, 0, (cudaStream_t)stream>>>(
      synth_key(seed, tensor_id), row0, rows, cols, qs, scales);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}
