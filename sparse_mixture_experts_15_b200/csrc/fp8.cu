// FP8 E4M3 quantisation for the routed experts of the LatentMoE layer
// ("Stable LatentMoE interactive demo document", SiTU-GLU: the soft caps keep
// the hidden product within beta_g * beta_u = 4 * 25 = 100, under E4M3's
// largest finite value 448, which is what lets the experts run in FP8).
//
// Row-wise scheme (OCP E4M3, round to nearest even, saturating at 448):
//   s = amax(row) / 448 (one fp32 division; 1 for an all-zero row)
//   code[c] = e4m3(x[c] / s) (one fp32 division per element)
// so that s * e4m3(code) approximates x and the row's largest magnitude maps
// to +-448.  Weights are quantised per output row, activations per token.
#include "common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float row_amax(const __nv_bfloat16* x, int cols, int lane) {
  float m = 0.0f;
  for (int c = lane * 8; c < cols; c += 256) {
    float v[8];
    load8(x + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
  }
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}
__device__ __forceinline__ float row_amax(const float* x, int cols, int lane) {
  float m = 0.0f;
  for (int c = lane * 8; c < cols; c += 256) {
    float v[8];
    load8(x + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
  }
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// One warp quantises one row of `cols` elements (cols % 8 == 0) into codes.
template <typename T>
__device__ __forceinline__ void quant_row(const T* x, int cols, int lane, uint8_t* codes,
                                          float* scale) {
  const float amax = row_amax(x, cols, lane);
  const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  for (int c = lane * 8; c < cols; c += 256) {
    float v[8];
    load8(x + c, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __fdiv_rn(v[i], s);
    *reinterpret_cast<uint2*>(codes + c) = make_uint2(e4m3x4_rn(v), e4m3x4_rn(v + 4));
  }
  if (lane == 0) *scale = s;
}

template <typename T>
__global__ void __launch_bounds__(256)
    quant_rows(const T* __restrict__ x, int64_t rows, int cols, uint8_t* __restrict__ codes,
               float* __restrict__ scales) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += ((int64_t)gridDim.x * blockDim.x) >> 5)
    quant_row(x + r * cols, cols, lane, codes + r * cols, scales + r);
}

// Grouped row r gets token perm_tok[r]'s row of x quantised: the gather of
// the expert path fused with the per-token quantisation (identical rows give
// identical codes and scales, so quantising after the gather equals
// quantising each token once and gathering codes and scales).
__global__ void __launch_bounds__(256)
    quant_gather(const __nv_bfloat16* __restrict__ x, int T, int cols,
                 const int32_t* __restrict__ perm_tok, const int32_t* __restrict__ offsets, int N,
                 int max_rows, uint8_t* __restrict__ codes, float* __restrict__ scales,
                 int* status) {
  pdl_wait();
  pdl_allow_next();
  int rows = offsets[N];
  if (rows < 0 || rows > max_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(status, MOE_ERR_BOUNDS);
    rows = rows < 0 ? 0 : max_rows;
  }
  const int lane = threadIdx.x & 31;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += (gridDim.x * blockDim.x) >> 5) {
    const int t = perm_tok[r];
    if (t < 0 || t >= T) {
      if (lane == 0) record_error(status, MOE_ERR_BOUNDS);
      continue;
    }
    quant_row(x + (size_t)t * cols, cols, lane, codes + (size_t)r * cols, scales + r);
  }
}

int warp_grid(int64_t warps) {
  int64_t b = (warps + 7) / 8;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b > 0 ? b : 1);
}

}  // namespace

int launch_quant_gather_e4m3(const moe_shape& s, int cols, const __nv_bfloat16* x,
                             const int32_t* perm_tok, const int32_t* offsets, uint8_t* codes,
                             float* scales, cudaStream_t st) {
  const int64_t max_rows = (int64_t)s.T * s.k;
  if (max_rows == 0) return MOE_OK;
  MOE_PREFER_SHARED((quant_gather));
  launch_pdl(quant_gather, dim3(warp_grid(max_rows)), dim3(256), 0, st, x, s.T, cols, perm_tok,
             offsets, s.N, (int)max_rows, codes, scales, status_word());
  return launch_status();
}

}  // namespace moe

extern "C" int moe_quantize_e4m3_rows(int64_t rows, int32_t cols, const void* x, int32_t x_dtype,
                                      uint8_t* codes, float* scales, void* stream) {
  using namespace moe;
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return MOE_ERR_INVALID_ARG;
  if (x_dtype != MOE_BF16 && x_dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes) ||
      (reinterpret_cast<uintptr_t>(scales) & 3u))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int grid = warp_grid(rows);
  if (x_dtype == MOE_BF16) {
    MOE_PREFER_SHARED((quant_rows<__nv_bfloat16>));
    launch_pdl(quant_rows<__nv_bfloat16>, dim3(grid), dim3(256), 0, st,
               static_cast<const __nv_bfloat16*>(x), rows, (int)cols, codes, scales);
  } else {
    MOE_PREFER_SHARED((quant_rows<float>));
    launch_pdl(quant_rows<float>, dim3(grid), dim3(256), 0, st, static_cast<const float*>(x),
               rows, (int)cols, codes, scales);
  }
  return launch_status();
}

extern "C" size_t moe_expert_ffn_e4m3_workspace_bytes(const moe_shape* shape) {
  if (!moe::shape_ok(shape) || shape->h <= 0) return 0;
  return moe::align_up((size_t)shape->T * shape->k * shape->h, 256);  // H as E4M3 codes
}

extern "C" int moe_expert_ffn_e4m3(const moe_shape* shape, int32_t width, const uint8_t* x_rows,
                                   const float* x_scale, const int32_t* offsets,
                                   const uint8_t* w_gate, const uint8_t* w_up,
                                   const uint8_t* w_down, const moe_e4m3_scales* scales,
                                   const moe_act* act, float* y_rows, void* ws, size_t ws_bytes,
                                   void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || !act || !scales || !offsets || !w_gate || !w_up || !w_down)
    return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (width <= 0 || width % 128 != 0 || s.h <= 0 || s.h % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (act->kind != MOE_ACT_SWIGLU &&
      !(act->kind == MOE_ACT_SITU_GLU && act->beta_gate > 0.0f && act->beta_up > 0.0f))
    return MOE_ERR_INVALID_ARG;
  if (!scales->gate_scale || !scales->up_scale || !scales->down_scale) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (!x_rows || !x_scale || !y_rows)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_expert_ffn_e4m3_workspace_bytes(shape)) return MOE_ERR_WORKSPACE;
  const int64_t R = (int64_t)s.T * s.k;
  if (R == 0) return MOE_OK;
  cudaStream_t st = as_stream(stream);
  TcF8 gu{{scales->gate_scale, scales->up_scale}, x_scale};
  int rc = tc_gateup(offsets, (int)R, s.N, x_rows, R, width, w_gate, w_up, s.h, *act, ws, s.h, 0,
                     st, &gu);
  if (rc != MOE_OK) return rc;
  TcF8 dn{{scales->down_scale, nullptr}, nullptr};
  TcSeg seg{w_down, (int64_t)s.N * width, s.h, 0, ws, R, s.h, 0};
  return tc_store(offsets, (int)R, s.N, width, &seg, 1, y_rows, MODE_STORE_F32, width, st, &dn);
}
