// Switch balancing statistics (tutorial "Mixture of Experts MoE: how sparse
// activation saves compute", §3.4): f_i (argmax share), P_i (mean router
// probability), N * sum f_i P_i (the auxiliary term without alpha), and the
// per-expert dispatch loads L_i of §3.6.
#include "common.cuh"

namespace moe {
namespace {

// Grid-stride over tokens; per-block partial sums in shared memory, then one
// global atomic per expert and block.  Counts are integers (exact); P is an
// fp32 sum whose order across blocks is not fixed (a statistic, compared with
// a tolerance).
__global__ void __launch_bounds__(256)
    stats_accumulate(const float* __restrict__ probs, const int32_t* __restrict__ top_idx, int T,
                     int N, int k, int32_t* __restrict__ argmax_cnt, int32_t* __restrict__ loads,
                     float* __restrict__ Psum, int* status) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ char smem[];
  int32_t* c_arg = reinterpret_cast<int32_t*>(smem);
  int32_t* c_load = c_arg + N;
  float* c_p = reinterpret_cast<float*>(c_load + N);
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    c_arg[i] = 0;
    c_load[i] = 0;
    c_p[i] = 0.0f;
  }
  __syncthreads();
  const int per_block = (T + gridDim.x - 1) / gridDim.x;
  const int tb = blockIdx.x * per_block, te = min(T, tb + per_block);
  for (int x = tb * k + threadIdx.x; x < te * k; x += blockDim.x) {
    const int e = top_idx[x];
    if (e < 0 || e >= N) {
      record_error(status, MOE_ERR_BOUNDS);
      continue;
    }
    atomicAdd(&c_load[e], 1);
    if (x % k == 0) atomicAdd(&c_arg[e], 1);
  }
  if (probs) {
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      float s = 0.0f;
      for (int t = tb; t < te; ++t) s += probs[(size_t)t * N + i];
      c_p[i] = s;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    atomicAdd(&argmax_cnt[i], c_arg[i]);
    atomicAdd(&loads[i], c_load[i]);
    if (probs) atomicAdd(&Psum[i], c_p[i]);
  }
}

__global__ void stats_finish(const int32_t* __restrict__ argmax_cnt,
                             const int32_t* __restrict__ loads_in, const float* __restrict__ Psum,
                             int T, int N, int has_p, float* __restrict__ f, float* __restrict__ P,
                             float* __restrict__ n_sum_fP, int32_t* __restrict__ loads) {
  pdl_wait();
  pdl_allow_next();
  __shared__ float red[32];
  float acc = 0.0f;
  const float inv_t = T > 0 ? 1.0f / (float)T : 0.0f;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const float fi = (float)argmax_cnt[i] * inv_t;
    const float pi = has_p ? Psum[i] * inv_t : 0.0f;
    if (f) f[i] = fi;
    if (P) P[i] = pi;
    if (loads) loads[i] = loads_in[i];
    acc += fi * pi;
  }
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
    if (n_sum_fP) n_sum_fP[0] = (float)N * s;
  }
}

// Tutorial §3.7: with the batch loads f held constant,
// dL_aux/dz_tj = c p_tj (f_j - sum_i f_i p_ti), c = alpha N / T.  One warp
// per token: lane l sums f_i p_ti over i = l, l + 32, ... in order, a
// butterfly adds the 32 partial sums, then each lane writes its experts.
__global__ void __launch_bounds__(256)
    aux_grad_kernel(const float* __restrict__ probs, const float* __restrict__ f, int T, int N,
                    float c, float* __restrict__ dz) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T;
       t += (gridDim.x * blockDim.x) >> 5) {
    const float* pt = probs + (size_t)t * N;
    float part = 0.0f;
    for (int i = lane; i < N; i += 32) part = __fmaf_rn(f[i], pt[i], part);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, o));
    for (int j = lane; j < N; j += 32)
      dz[(size_t)t * N + j] = __fmul_rn(__fmul_rn(c, pt[j]), __fsub_rn(f[j], part));
  }
}

}  // namespace

size_t aux_stats_ws_bytes(int32_t N) { return align_up((size_t)N * 12, 256); }

int launch_aux_stats(int32_t T, int32_t N, int32_t k, const float* probs, const int32_t* top_idx,
                     float* f, float* P, float* n_sum_fP, int32_t* loads, void* ws,
                     cudaStream_t st) {
  int32_t* c_arg = static_cast<int32_t*>(ws);
  int32_t* c_load = c_arg + N;
  float* c_p = reinterpret_cast<float*>(c_load + N);
  cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)N * 12, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (T > 0) {
    int blocks = (T + 63) / 64;
    if (blocks > 148) blocks = 148;
    MOE_PREFER_SHARED((stats_accumulate));
    launch_pdl(stats_accumulate, dim3(blocks), dim3(256), (size_t)N * 12, st, probs, top_idx, T, N, k, c_arg, c_load,
                                                          c_p, status_word());
  }
  MOE_PREFER_SHARED((stats_finish));
  launch_pdl(stats_finish, dim3(1), dim3(1024), 0, st, c_arg, c_load, c_p, T, N, probs != nullptr, f, P, n_sum_fP,
                                   loads);
  return launch_status();
}

}  // namespace moe

extern "C" size_t moe_aux_stats_workspace_bytes(int32_t N) {
  return N > 0 ? moe::aux_stats_ws_bytes(N) : 0;
}

extern "C" int moe_aux_stats(int32_t T, int32_t N, int32_t k, const float* probs,
                             const int32_t* top_idx, float* f, float* P, float* n_sum_fP,
                             int32_t* loads, void* ws, size_t ws_bytes, void* stream) {
  using namespace moe;
  if (T < 0 || N <= 0 || N > 1024 || k <= 0 || k > N) return MOE_ERR_INVALID_ARG;
  if (T > 0 && !top_idx) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < aux_stats_ws_bytes(N)) return MOE_ERR_WORKSPACE;
  return launch_aux_stats(T, N, k, probs, top_idx, f, P, n_sum_fP, loads, ws, as_stream(stream));
}

extern "C" int moe_aux_grad(int32_t T, int32_t N, float alpha, const float* probs, const float* f,
                            float* dz, void* stream) {
  using namespace moe;
  if (T < 0 || N <= 0 || N > 1024) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!probs || !f || !dz) return MOE_ERR_INVALID_ARG;
  const float c = (float)((double)alpha * (double)N / (double)T);
  int blocks = (T + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  MOE_PREFER_SHARED((aux_grad_kernel));
  launch_pdl(aux_grad_kernel, dim3(blocks), dim3(256), 0, as_stream(stream), probs, f, T, N, c, dz);
  return launch_status();
}
