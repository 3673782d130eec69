// Grouped SwiGLU experts in fp32 on the SIMT cores, for fp32 layers (the
// tensor cores have no fp32 mode of full fp32 accuracy; TF32 would miss a
// 1e-4 relative tolerance).  Tutorial "Mixture of Experts MoE: how sparse
// activation saves compute", §3.1 equation F:
//   F(u) = W_down (SiLU(W_gate u) * W_up u).
// One block per grouped row: the row is staged in shared memory and each
// thread produces hidden units (then output features) with fp32 FMAs.
#include "common.cuh"

namespace moe {
namespace {

// Expert of grouped row r: the e with offsets[e] <= r < offsets[e+1].
__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int N, int r) {
  int lo = 0, hi = N;  // invariant: offsets[lo] <= r < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float act_fn(float g, float v, const moe_act& a) {
  if (a.kind == MOE_ACT_SITU_GLU) {
    g = a.beta_gate * tanhf(g / a.beta_gate);
    v = a.beta_up * tanhf(v / a.beta_up);
  }
  return silu(g) * v;
}

__global__ void __launch_bounds__(256)
    ffn_gateup_simt(const float* __restrict__ x_rows, int width, int h,
                    const int32_t* __restrict__ offsets, int N, const float* __restrict__ wg,
                    const float* __restrict__ wu, moe_act act, float* __restrict__ H) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ float xs[];
  const int r = blockIdx.x;
  if (r >= offsets[N]) return;
  const int e = expert_of_row(offsets, N, r);
  for (int c = threadIdx.x; c < width; c += blockDim.x) xs[c] = x_rows[(size_t)r * width + c];
  __syncthreads();
  const float* wge = wg + (size_t)e * h * width;
  const float* wue = wu + (size_t)e * h * width;
  for (int i = threadIdx.x; i < h; i += blockDim.x) {
    float g = 0.0f, v = 0.0f;
    const float* a = wge + (size_t)i * width;
    const float* b = wue + (size_t)i * width;
    for (int c = 0; c < width; ++c) {
      g = __fmaf_rn(a[c], xs[c], g);
      v = __fmaf_rn(b[c], xs[c], v);
    }
    H[(size_t)r * h + i] = act_fn(g, v, act);
  }
}

__global__ void __launch_bounds__(256)
    ffn_down_simt(const float* __restrict__ H, int h, int width,
                  const int32_t* __restrict__ offsets, int N, const float* __restrict__ wd,
                  float* __restrict__ y_rows) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ float hs[];
  const int r = blockIdx.x;
  if (r >= offsets[N]) return;
  const int e = expert_of_row(offsets, N, r);
  for (int c = threadIdx.x; c < h; c += blockDim.x) hs[c] = H[(size_t)r * h + c];
  __syncthreads();
  const float* wde = wd + (size_t)e * width * h;
  for (int m = threadIdx.x; m < width; m += blockDim.x) {
    float acc = 0.0f;
    const float* a = wde + (size_t)m * h;
    for (int i = 0; i < h; ++i) acc = __fmaf_rn(a[i], hs[i], acc);
    y_rows[(size_t)r * width + m] = acc;
  }
}

}  // namespace

size_t ffn_simt_ws_bytes(const moe_shape& s) {
  return align_up((size_t)s.T * s.k * s.h * 4, 256);
}

int launch_ffn_simt(const moe_shape& s, int32_t width, const float* x_rows, const int32_t* offsets,
                    const float* w_gate, const float* w_up, const float* w_down,
                    const moe_act& act, float* y_rows, void* ws, cudaStream_t st) {
  const int64_t max_rows = (int64_t)s.T * s.k;
  if (max_rows == 0) return MOE_OK;
  float* H = static_cast<float*>(ws);
  MOE_PREFER_SHARED((ffn_gateup_simt));
  launch_pdl(ffn_gateup_simt, dim3((unsigned)max_rows), dim3(256), (size_t)width * 4, st, x_rows, width, s.h, offsets,
                                                                       s.N, w_gate, w_up, act, H);
  MOE_PREFER_SHARED((ffn_down_simt));
  launch_pdl(ffn_down_simt, dim3((unsigned)max_rows), dim3(256), (size_t)s.h * 4, st, H, s.h, width, offsets, s.N,
                                                                  w_down, y_rows);
  return launch_status();
}

}  // namespace moe
