// Quantile balancing of the expert biases ("Stable LatentMoE interactive demo
// document", Quantile Balancing).  With every token's top-k cutoff a_i held
// fixed, expert j takes token i iff s_ij + b_j >= a_i, i.e. iff
// b_j >= required_ij = a_i - s_ij, so the bias that gives expert j exactly q
// tokens is the q-th smallest required_ij (one step, no learning rate).  The
// page contrasts the exact quantile with a histogram estimate; both are here.
//
//   qb_cutoffs   one warp per token: the selection scores s_ij + b_j sit in
//                registers (a lane holds experts lane, lane + 32, ...), k
//                rounds of a warp-wide arg-max leave a_i, the k-th largest.
//   qb_select    one block per expert: required_ij for all tokens as
//                order-preserving 32-bit keys in shared memory; the q-th
//                smallest by a 4-pass radix select (8 bits per pass, warp-
//                aggregated shared-memory counts); the load
//                #{i : required_ij <= b_j}; and, when asked, the histogram
//                estimate (bins over [min, max], the upper edge of the bin
//                where the running count reaches q).
// Every arithmetic step is one fp32 operation in a fixed order, so the exact
// bias, the cutoffs and the histogram estimate are reproducible bit for bit.
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kQBThreads = 256;
constexpr int kQBMaxT = 32768;  // required keys of one expert in shared memory
constexpr int kQBMaxBins = 4096;
constexpr int kQBMaxK = 32;

// float <-> key whose unsigned order is the float order (-0 just below +0)
__device__ __forceinline__ uint32_t fkey(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float unkey(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int MPER>
__global__ void __launch_bounds__(256)
    qb_cutoffs(const float* __restrict__ s, const float* __restrict__ bias, int T, int N, int k,
               float* __restrict__ a) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float v[MPER];
#pragma unroll
  for (int m = 0; m < MPER; ++m) {
    const int j = lane + 32 * m;
    v[m] = j < N ? (bias ? __fadd_rn(s[(size_t)t * N + j], bias[j]) : s[(size_t)t * N + j])
                 : -FLT_MAX;
  }
  uint32_t taken = 0;  // bit m: v[m] already ranked
  float kth = 0.0f;
  for (int r = 0; r < k; ++r) {
    float bv = 0.0f;
    int bj = INT_MAX;
#pragma unroll
    for (int m = 0; m < MPER; ++m) {
      const int j = lane + 32 * m;
      if (j < N && !((taken >> m) & 1u) && (bj == INT_MAX || v[m] > bv)) {
        bv = v[m];
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {  // larger value, then lower index
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (oj != INT_MAX && (bj == INT_MAX || ov > bv || (ov == bv && oj < bj))) {
        bv = ov;
        bj = oj;
      }
    }
    if (bj != INT_MAX && (bj & 31) == lane) taken |= 1u << (bj >> 5);
    kth = bv;
  }
  if (lane == 0) a[t] = kth;
}

// Counts of 8-bit digits of the candidate keys (those matching `prefix` under
// `mask`), one shared atomic per distinct digit per warp.
__device__ __forceinline__ void digit_counts(const uint32_t* keys, int T, uint32_t prefix,
                                             uint32_t mask, int shift, int* hist) {
  const int lane = threadIdx.x & 31;
  const int rounds = (T + blockDim.x - 1) / blockDim.x;
  for (int r = 0; r < rounds; ++r) {
    const int i = r * blockDim.x + threadIdx.x;
    int digit = -1;
    if (i < T) {
      const uint32_t key = keys[i];
      if ((key & mask) == prefix) digit = (int)((key >> shift) & 0xFFu);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, digit);
    if (digit >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
  }
}

__global__ void __launch_bounds__(kQBThreads)
    qb_select(const float* __restrict__ s, const float* __restrict__ a, int T, int N, int q,
              int bins, float* __restrict__ b_exact, float* __restrict__ b_hist,
              int32_t* __restrict__ loads) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ __align__(16) uint32_t keys[];  // [T]
  __shared__ int hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_rem, s_cnt;
  __shared__ float s_red[2][kQBThreads / 32];
  int* bin_cnt = reinterpret_cast<int*>(keys + T);  // [bins]
  const int j = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // required biases a_i - s_ij of column j: eight strided loads in flight per thread
  for (int i0 = tid; i0 < T; i0 += 8 * blockDim.x) {
    float sv[8], av[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      sv[u] = i < T ? s[(size_t)i * N + j] : 0.0f;
      av[u] = i < T ? a[i] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * (int)blockDim.x;
      if (i < T) keys[i] = fkey(__fsub_rn(av[u], sv[u]));
    }
  }
  if (tid == 0) {
    s_prefix = 0;
    s_rem = q;
    s_cnt = 0;
  }
  __syncthreads();
  // ---- exact: radix select of the q-th smallest key, most significant digit first
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t mask = pass == 0 ? 0u : 0xFFFFFFFFu << (32 - 8 * pass);
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    digit_counts(keys, T, s_prefix, mask, shift, hist);
    __syncthreads();
    if (warp == 0) {
      // the first digit whose cumulative count reaches rem (255 at most),
      // and rem less the counts before it: lane l scans digits 8l .. 8l+7,
      // a warp prefix sum finds the lane, that lane finds the digit
      int v[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[i] = hist[lane * 8 + i];
        sum += v[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
      }
      const int rem = s_rem;
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= rem);
      const int L = hit ? __ffs(hit) - 1 : 31;
      if (lane == L) {
        int r = rem - (incl - sum), dgt = lane * 8;
        for (int i = 0; i < 8; ++i, ++dgt) {
          if (dgt == 255 || v[i] >= r) break;
          r -= v[i];
        }
        s_rem = r;
        s_prefix |= (uint32_t)dgt << shift;
      }
    }
    __syncthreads();
  }
  float bq = unkey(s_prefix);
  if (bq == 0.0f) bq = 0.0f;  // a zero bias is returned as +0
  // ---- load: tokens whose required bias is at most b_j
  int c = 0;
  for (int i = tid; i < T; i += blockDim.x) c += unkey(keys[i]) <= bq;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) atomicAdd(&s_cnt, c);
  // ---- histogram estimate
  float lo = FLT_MAX, hi = -FLT_MAX;
  if (b_hist) {
    for (int i = tid; i < T; i += blockDim.x) {
      const float v = unkey(keys[i]);
      lo = fminf(lo, v);
      hi = fmaxf(hi, v);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      s_red[0][warp] = lo;
      s_red[1][warp] = hi;
    }
    for (int i = tid; i < bins; i += blockDim.x) bin_cnt[i] = 0;
  }
  __syncthreads();
  if (tid == 0) {
    b_exact[j] = bq;
    if (loads) loads[j] = s_cnt;
  }
  if (!b_hist) return;
  lo = s_red[0][0];
  hi = s_red[1][0];
  for (int w = 1; w < kQBThreads / 32; ++w) {
    lo = fminf(lo, s_red[0][w]);
    hi = fmaxf(hi, s_red[1][w]);
  }
  if (!(hi > lo)) {
    if (tid == 0) b_hist[j] = lo == 0.0f ? 0.0f : lo;
    return;
  }
  const float range = __fsub_rn(hi, lo);
  const float scale = __fdiv_rn((float)bins, range);
  const float width = __fdiv_rn(range, (float)bins);
  for (int i = tid; i < T; i += blockDim.x) {
    const float x = __fmul_rn(__fsub_rn(unkey(keys[i]), lo), scale);
    int cb = __float2int_rz(x);
    if (cb > bins - 1) cb = bins - 1;
    atomicAdd(&bin_cnt[cb], 1);
  }
  __syncthreads();
  if (warp == 0) {
    // the first bin whose cumulative count reaches q (the last bin at most):
    // 32 bins per step, a warp prefix sum with the running total carried
    int cb = bins - 1, carry = 0;
    for (int base = 0; base < bins; base += 32) {
      const int c = base + lane < bins ? bin_cnt[base + lane] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int nb = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += nb;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, base + lane < bins && carry + incl >= q);
      if (hit) {
        cb = base + __ffs(hit) - 1;
        break;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) b_hist[j] = __fadd_rn(lo, __fmul_rn((float)(cb + 1), width));
  }
}

size_t select_smem(int T, int bins) { return (size_t)T * 4 + (size_t)bins * 4; }

}  // namespace
}  // namespace moe

extern "C" size_t moe_quantile_balance_workspace_bytes(int32_t T, int32_t N) {
  if (T < 1 || N < 1) return 0;
  return moe::align_up((size_t)T * 4, 256);
}

extern "C" int moe_quantile_balance(int32_t T, int32_t N, int32_t k, const float* scores,
                                    const float* bias, int32_t q, int32_t bins, float* cutoff,
                                    float* bias_exact, float* bias_hist, int32_t* loads, void* ws,
                                    size_t ws_bytes, void* stream) {
  using namespace moe;
  if (T < 1 || T > kQBMaxT || N < 1 || N > 1024 || k < 1 || k > N || k > kQBMaxK || q < 1 ||
      q > T || bins < 0 || bins > kQBMaxBins || (bias_hist && bins < 1))
    return MOE_ERR_INVALID_ARG;
  if (!scores || !bias_exact) return MOE_ERR_INVALID_ARG;
  float* a = cutoff;
  if (!a) {
    if (!ws || ws_bytes < moe_quantile_balance_workspace_bytes(T, N)) return MOE_ERR_WORKSPACE;
    a = static_cast<float*>(ws);
  }
  cudaStream_t st = as_stream(stream);
  const int per = (N + 31) / 32;
  const dim3 grid((unsigned)((T + 7) / 8));
#define MOE_QB_CUT(M)                                                                      \
  do {                                                                                     \
    MOE_PREFER_SHARED((qb_cutoffs<M>));                                                    \
    launch_pdl(qb_cutoffs<M>, grid, dim3(256), 0, st, scores, bias, T, N, k, a);           \
  } while (0)
  if (per <= 1) MOE_QB_CUT(1);
  else if (per <= 2) MOE_QB_CUT(2);
  else if (per <= 4) MOE_QB_CUT(4);
  else if (per <= 8) MOE_QB_CUT(8);
  else if (per <= 16) MOE_QB_CUT(16);
  else MOE_QB_CUT(32);
#undef MOE_QB_CUT
  const size_t smem = select_smem(T, bias_hist ? bins : 0);
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (needs_setup(configured, dev)) {
    if (cudaFuncSetAttribute(qb_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)select_smem(kQBMaxT, kQBMaxBins)) != cudaSuccess)
      return MOE_ERR_CUDA;
    mark_setup(configured, dev);
  }
  MOE_PREFER_SHARED((qb_select));
  launch_pdl(qb_select, dim3((unsigned)N), dim3(kQBThreads), smem, st, scores,
             static_cast<const float*>(a), T, N, q, bias_hist ? bins : 0, bias_exact, bias_hist,
             loads);
  return launch_status();
}
