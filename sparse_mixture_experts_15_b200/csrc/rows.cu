// Row movement around the experts (tutorial "Mixture of Experts MoE: how
// sparse activation saves compute", §3.6: split tokens into per-expert
// [L_i, d] rows, then add the results back into [T, d]):
//   gather:  x_rows[r] = u[perm_tok[r]]
//   combine: y[t] = sum_s a_{t,s} y_rows[row_of[t][s]]  (§3.2 eq. y)
#include "common.cuh"

namespace moe {
namespace {

// One warp per grouped row, 16-byte vectors (row bytes are a multiple of 16).
__global__ void __launch_bounds__(256)
    gather_rows(const uint4* __restrict__ u, int vec_per_row, const int32_t* __restrict__ perm_tok,
                const int32_t* __restrict__ offsets, int N, int T, int max_rows,
                uint4* __restrict__ x_rows, int* status) {
  pdl_wait();
  pdl_allow_next();
  int rows = offsets[N];
  if (rows < 0 || rows > max_rows) {  // x_rows and perm_tok hold T*k rows
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
    const uint4* src = u + (size_t)t * vec_per_row;
    uint4* dst = x_rows + (size_t)r * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) dst[v] = src[v];
  }
}

template <typename TY>
__device__ __forceinline__ void store4(TY* y, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* y, float4 v) {
  *reinterpret_cast<float4*>(y) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* y, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 o;
  o.x = *reinterpret_cast<uint32_t*>(&a);
  o.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(y) = o;
}
template <>
__device__ __forceinline__ void store4<__half>(__half* y, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
  uint2 o;
  o.x = *reinterpret_cast<uint32_t*>(&a);
  o.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(y) = o;
}

// One warp per token; slots are added in ascending s (fixed order).
template <typename TY>
__global__ void __launch_bounds__(256)
    combine_rows(const float4* __restrict__ y_rows, int width4, const int32_t* __restrict__ row_of,
                 const float* __restrict__ top_w, int T, int k, TY* __restrict__ y,
                 int* status) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T;
       t += (gridDim.x * blockDim.x) >> 5) {
    for (int c = lane; c < width4; c += 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < k; ++s) {
        const int r = row_of[(size_t)t * k + s];
        if (r < 0) continue;
        if (r >= T * k) {  // y_rows holds T*k rows
          record_error(status, MOE_ERR_BOUNDS);
          continue;
        }
        const float a = top_w[(size_t)t * k + s];
        const float4 v = y_rows[(size_t)r * width4 + c];
        acc.x = __fmaf_rn(a, v.x, acc.x);
        acc.y = __fmaf_rn(a, v.y, acc.y);
        acc.z = __fmaf_rn(a, v.z, acc.z);
        acc.w = __fmaf_rn(a, v.w, acc.w);
      }
      store4<TY>(y + ((size_t)t * width4 + c) * 4, acc);
    }
  }
}

// One warp per token; rows already carry their weights (fp32 a * F(u)), the
// kept slots are added in ascending s in fp32 and rounded once.  The token's
// k (<= 32) slot row indices are read once into shared memory; a lane loads
// two slots' rows for four of its columns before adding them, so a warp has
// eight loads per lane in flight.
template <typename TY>
__global__ void __launch_bounds__(256)
    combine_weighted(const float4* __restrict__ rows, int width4,
                     const int32_t* __restrict__ row_of, int T, int k, TY* __restrict__ y,
                     int* status) {
  pdl_wait();
  pdl_allow_next();
  __shared__ int srow[256 / 32][32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T;
       t += (gridDim.x * blockDim.x) >> 5) {
    int r = lane < k ? row_of[(size_t)t * k + lane] : -1;
    if (r >= T * k) {  // rows holds T*k rows
      record_error(status, MOE_ERR_BOUNDS);
      r = -1;
    }
    srow[wib][lane] = r;
    __syncwarp();
    // four columns per lane at a time (c0 + 32 q), two slots per round: the
    // eight row loads of a round are in flight together
    for (int c0 = lane; c0 < width4; c0 += 32 * 4) {
      float4 acc[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < k; s0 += 2) {
        float4 v[2][4];
        int rs[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          rs[j] = s0 + j < k ? srow[wib][s0 + j] : -1;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (rs[j] >= 0 && c0 + 32 * q < width4)
              v[j][q] = rows[(size_t)rs[j] * width4 + c0 + 32 * q];
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (rs[j] >= 0 && c0 + 32 * q < width4) {
              acc[q].x += v[j][q].x;
              acc[q].y += v[j][q].y;
              acc[q].z += v[j][q].z;
              acc[q].w += v[j][q].w;
            }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (c0 + 32 * q < width4) store4<TY>(y + ((size_t)t * width4 + c0 + 32 * q) * 4, acc[q]);
    }
    __syncwarp();  // srow is rewritten for the warp's next token
  }
}

int grid_cap(int64_t warps) {
  int64_t b = (warps + 7) / 8;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b > 0 ? b : 1);
}

}  // namespace

int launch_gather(const moe_shape& s, int32_t width, const void* u, int32_t dtype,
                  const int32_t* perm_tok, const int32_t* offsets, void* x_rows, cudaStream_t st) {
  const int vec = (int)((size_t)width * dtype_bytes(dtype) / 16);
  const int64_t max_rows = (int64_t)s.T * s.k;
  if (max_rows == 0) return MOE_OK;
  MOE_PREFER_SHARED((gather_rows));
  launch_pdl(gather_rows, dim3(grid_cap(max_rows)), dim3(256), 0, st, static_cast<const uint4*>(u), vec, perm_tok,
             offsets, s.N, s.T, (int)max_rows, static_cast<uint4*>(x_rows), status_word());
  return launch_status();
}

int launch_combine(const moe_shape& s, int32_t width, const float* y_rows, const int32_t* row_of,
                   const float* top_w, void* y, int32_t y_dtype, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  const int w4 = width / 4;
  const int grid = grid_cap(s.T);
  const float4* yr = reinterpret_cast<const float4*>(y_rows);
  if (y_dtype == MOE_F32) {
    MOE_PREFER_SHARED((combine_rows<float>));
    launch_pdl(combine_rows<float>, dim3(grid), dim3(256), 0, st, yr, w4, row_of, top_w, s.T, s.k,
               static_cast<float*>(y), status_word());
  } else if (y_dtype == MOE_BF16) {
    MOE_PREFER_SHARED((combine_rows<__nv_bfloat16>));
    launch_pdl(combine_rows<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, yr, w4, row_of, top_w,
               s.T, s.k, static_cast<__nv_bfloat16*>(y), status_word());
  } else {
    MOE_PREFER_SHARED((combine_rows<__half>));
    launch_pdl(combine_rows<__half>, dim3(grid), dim3(256), 0, st, yr, w4, row_of, top_w, s.T, s.k,
               static_cast<__half*>(y), status_word());
  }
  return launch_status();
}

int launch_combine_weighted(const moe_shape& s, int32_t width, const float* rows,
                            const int32_t* row_of, void* y, int32_t y_dtype, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  const int w4 = width / 4;
  const int grid = grid_cap(s.T);
  const float4* r = reinterpret_cast<const float4*>(rows);
  if (y_dtype == MOE_F32) {
    MOE_PREFER_SHARED((combine_weighted<float>));
    launch_pdl(combine_weighted<float>, dim3(grid), dim3(256), 0, st, r, w4, row_of, s.T, s.k,
               static_cast<float*>(y), status_word());
  } else if (y_dtype == MOE_BF16) {
    MOE_PREFER_SHARED((combine_weighted<__nv_bfloat16>));
    launch_pdl(combine_weighted<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, r, w4, row_of,
               s.T, s.k, static_cast<__nv_bfloat16*>(y), status_word());
  } else {
    MOE_PREFER_SHARED((combine_weighted<__half>));
    launch_pdl(combine_weighted<__half>, dim3(grid), dim3(256), 0, st, r, w4, row_of, s.T, s.k,
               static_cast<__half*>(y), status_word());
  }
  return launch_status();
}

}  // namespace moe

extern "C" int moe_gather(const moe_shape* shape, int32_t width, const void* u, int32_t dtype,
                          const int32_t* perm_tok, const int32_t* offsets, void* x_rows,
                          void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || !valid_act_dtype(dtype) || width <= 0 || width % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (!offsets || (shape->T > 0 && (!u || !perm_tok || !x_rows))) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(x_rows)) return MOE_ERR_INVALID_ARG;
  return launch_gather(*shape, width, u, dtype, perm_tok, offsets, x_rows, as_stream(stream));
}

extern "C" int moe_combine(const moe_shape* shape, int32_t width, const float* y_rows,
                           const int32_t* row_of, const float* top_w, void* y, int32_t y_dtype,
                           void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || !valid_act_dtype(y_dtype) || width <= 0 || width % 8 != 0)
    return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!y_rows || !row_of || !top_w || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_rows) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  return launch_combine(*shape, width, y_rows, row_of, top_w, y, y_dtype, as_stream(stream));
}
