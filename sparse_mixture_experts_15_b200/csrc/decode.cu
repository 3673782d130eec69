// Small-batch decode path with q4_0 experts.
//
// Deployment notes "Kestrel-MCU notes 13", §2 and §4: per layer the router
// GEMV picks the top-k experts, and only the selected experts' gate/up/down
// weights are read ("lookup loading"), stored as q4_0 (32-value blocks, one
// fp16 scale s, 4-bit q, w = (q - 8) s).  The tutorial "Mixture of Experts
// MoE: how sparse activation saves compute" §3.1-§3.2 fixes the arithmetic.
// Layers chain as u_{l+1} = fp16(u_l + y_l).
//
// Per layer two phases, each one launch:
//   decode_gateup (grid = experts x 16-row hidden slices): every CTA stages
//     u and W_route in shared memory and routes all T tokens itself (the
//     router is tiny: N x d fp32), leaves at once if
//     no token selected its expert (so unselected weights are never read),
//     otherwise dequantises its 16 gate + 16 up rows in registers and writes
//     H[e][t][slice] = SiLU(g) * u for its tokens.
//   decode_down (grid = 32-row slices of the output): stages the H row of
//     every (token, slot) in shared memory; for every selected expert,
//     dequantises its down rows once and forms each (token, slot) dot with
//     H, then sums the slots in order: y = sum_s a_s W_down H,
//     u_next = fp16(u + y).
// Weights are streamed with 16-byte loads and dequantised in registers.
#include <cfloat>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kRowsA = 16;    // hidden rows per gate/up CTA (x2: gate and up)
constexpr int kRowsB = 32;    // output rows per down CTA
constexpr int kMaxT = 32;     // decode batch limit
constexpr int kMaxN = 64;     // expert limit of the decode kernels

__device__ __forceinline__ float f16f(uint16_t c) { return __half2float(__ushort_as_half(c)); }

// 32 weights of one q4_0 block: byte j -> element j (low nibble), j+16 (high).
__device__ __forceinline__ void dequant_block(const uint8_t* qs, uint16_t scale, float* w) {
  const uint4 raw = *reinterpret_cast<const uint4*>(qs);
  const float s = f16f(scale);
  const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t byte = (wd[i] >> (8 * b)) & 0xFFu;
      w[4 * i + b] = (float)((int)(byte & 0xFu) - 8) * s;
      w[16 + 4 * i + b] = (float)((int)(byte >> 4) - 8) * s;
    }
  }
}

// 16-byte global -> shared copies issued without waiting (LDGSTS); one wait
// afterwards pays a single memory latency for the whole staging.
__device__ __forceinline__ void cp16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Copies rows x row_bytes (multiple of 16) from gmem (row stride g_stride
// bytes) to smem rows of s_stride bytes, all threads of the CTA cooperating.
__device__ __forceinline__ void stage_rows(char* smem, int s_stride, const char* gmem,
                                           size_t g_stride, int rows, int row_bytes) {
  const int per_row = row_bytes / 16;
  for (int i = threadIdx.x; i < rows * per_row; i += blockDim.x) {
    const int r = i / per_row, c = i - r * per_row;
    cp16(smem + (size_t)r * s_stride + c * 16, gmem + r * g_stride + (size_t)c * 16);
  }
}

// Routing of all T tokens inside one CTA from u_s [T] rows (fp16, row stride
// us_ld elements) and w_s [N] rows (fp32, stride ws_ld), both staged in
// shared memory with a 16-byte pad per row so the threads of a warp
// (consecutive (t, i) pairs) hit distinct banks.  z is the sequential fp32
// FMA chain over j (the order the oracle uses); ties go to the lower expert
// index.  Leaves sel[t][s] and aw[t][s] in shared memory.
__device__ void route_in_cta(const __half* u_s, int us_ld, const float* w_s, int ws_ld, int T,
                             int d, int N, int k, int renorm, const float* __restrict__ bias,
                             float* z, int* sel, float* aw) {
  const int pairs = T * N;
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    const int t = p / N, i = p - t * N;
    const __half2* ut = reinterpret_cast<const __half2*>(u_s + (size_t)t * us_ld);
    const float2* wi = reinterpret_cast<const float2*>(w_s + (size_t)i * ws_ld);
    float a = 0.0f;
#pragma unroll 8
    for (int j = 0; j < d / 2; ++j) {
      const float2 x = __half22float2(ut[j]);
      const float2 v = wi[j];
      a = __fmaf_rn(v.x, x.x, a);
      a = __fmaf_rn(v.y, x.y, a);
    }
    z[p] = bias ? __fadd_rn(a, bias[i]) : a;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const float* zt = z + t * N;
    float zmax = -FLT_MAX;
    for (int i = 0; i < N; ++i) zmax = fmaxf(zmax, zt[i]);
    float den = 0.0f;
    for (int i = 0; i < N; ++i) den += expf(zt[i] - zmax);
    uint64_t taken = 0;
    float ps = 0.0f;
    for (int s = 0; s < k; ++s) {
      int bi = -1;
      for (int i = 0; i < N; ++i)
        if (!((taken >> i) & 1ull) && (bi < 0 || zt[i] > zt[bi])) bi = i;
      taken |= 1ull << bi;
      sel[t * k + s] = bi;
      aw[t * k + s] = expf(zt[bi] - zmax) / den;
      ps += aw[t * k + s];
    }
    if (renorm)
      for (int s = 0; s < k; ++s) aw[t * k + s] /= ps;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(128)
    decode_gateup(const __half* __restrict__ u, int T, int d, int N, int k, int h, int renorm,
                  const float* __restrict__ w_route, const float* __restrict__ bias,
                  const uint8_t* __restrict__ gq, const uint16_t* __restrict__ gs,
                  const uint8_t* __restrict__ uq, const uint16_t* __restrict__ us,
                  float* __restrict__ H, int32_t* __restrict__ top_idx, float* __restrict__ top_w) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ __align__(16) char dyn[];
  const int us_ld = d + 8, ws_ld = d + 4, nb = d / 32;
  __half* u_s = reinterpret_cast<__half*>(dyn);                          // [T][d+8]
  float* w_s = reinterpret_cast<float*>(dyn + (size_t)T * us_ld * 2);     // [N][d+4]
  uint8_t* q_s = reinterpret_cast<uint8_t*>(w_s + (size_t)N * ws_ld);     // [32][d/2]
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(q_s + 2 * kRowsA * (d / 2));  // [32][d/32]
  __shared__ float z[kMaxT * kMaxN];
  __shared__ int sel[kMaxT * 8];
  __shared__ float aw[kMaxT * 8];
  __shared__ int toks[kMaxT];
  __shared__ int ntok;
  __shared__ float gu[2 * kRowsA][kMaxT + 1];
  const int slices = h / kRowsA;
  const int e = blockIdx.x / slices, slice = blockIdx.x - e * slices;
  stage_rows(reinterpret_cast<char*>(u_s), us_ld * 2, reinterpret_cast<const char*>(u),
             (size_t)d * 2, T, d * 2);
  stage_rows(reinterpret_cast<char*>(w_s), ws_ld * 4, reinterpret_cast<const char*>(w_route),
             (size_t)d * 4, N, d * 4);
  cp_wait_all();
  __syncthreads();
  route_in_cta(u_s, us_ld, w_s, ws_ld, T, d, N, k, renorm, bias, z, sel, aw);
  if (blockIdx.x == 0) {
    for (int x = threadIdx.x; x < T * k; x += blockDim.x) {
      top_idx[x] = sel[x];
      if (top_w) top_w[x] = aw[x];
    }
  }
  if (threadIdx.x == 0) {
    int n = 0;
    for (int t = 0; t < T; ++t) {
      bool hit = false;
      for (int s = 0; s < k; ++s) hit |= sel[t * k + s] == e;
      if (hit) toks[n++] = t;
    }
    ntok = n;
  }
  __syncthreads();
  const int n = ntok;
  if (n == 0) return;  // expert not selected: its weights are never read

  // stage this CTA's 16 gate + 16 up rows (q4 bytes and scales) in one go
  const size_t row_g = (size_t)e * h + slice * kRowsA;
  stage_rows(reinterpret_cast<char*>(q_s), d / 2, reinterpret_cast<const char*>(gq + row_g * (d / 2)),
             d / 2, kRowsA, d / 2);
  stage_rows(reinterpret_cast<char*>(q_s + kRowsA * (d / 2)), d / 2,
             reinterpret_cast<const char*>(uq + row_g * (d / 2)), d / 2, kRowsA, d / 2);
  if (nb * 2 >= 16) {
    stage_rows(reinterpret_cast<char*>(sc_s), nb * 2,
               reinterpret_cast<const char*>(gs + row_g * nb), (size_t)nb * 2, kRowsA, nb * 2);
    stage_rows(reinterpret_cast<char*>(sc_s + kRowsA * nb), nb * 2,
               reinterpret_cast<const char*>(us + row_g * nb), (size_t)nb * 2, kRowsA, nb * 2);
  } else {
    for (int i = threadIdx.x; i < 2 * kRowsA * nb; i += blockDim.x) {
      const int r = i / nb, c = i - r * nb;
      sc_s[i] = (r < kRowsA ? gs : us)[(row_g + (r % kRowsA)) * nb + c];
    }
  }
  cp_wait_all();
  __syncthreads();

  // (row, token) dots: consecutive threads take consecutive tokens of the
  // same weight row (the row's bytes are a shared-memory broadcast).
  for (int p = threadIdx.x; p < 2 * kRowsA * n; p += blockDim.x) {
    const int r = p / n, i = p - r * n;
    const uint8_t* q = q_s + (size_t)r * (d / 2);
    const uint16_t* sc = sc_s + (size_t)r * nb;
    const __half2* ut = reinterpret_cast<const __half2*>(u_s + (size_t)toks[i] * us_ld);
    float a0 = 0.0f, a1 = 0.0f;
    for (int bb = 0; bb < nb; ++bb) {
      float w[32];
      dequant_block(q + bb * 16, sc[bb], w);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float2 x = __half22float2(ut[bb * 16 + c]);
        a0 = fmaf(w[2 * c], x.x, a0);
        a1 = fmaf(w[2 * c + 1], x.y, a1);
      }
    }
    gu[r][i] = a0 + a1;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < n * kRowsA; x += blockDim.x) {
    const int i = x / kRowsA, r = x - i * kRowsA;
    H[((size_t)e * T + toks[i]) * h + slice * kRowsA + r] = silu(gu[r][i]) * gu[kRowsA + r][i];
  }
}

__global__ void __launch_bounds__(128)
    decode_down(const __half* __restrict__ u, int T, int d, int N, int k, int h,
                const int32_t* __restrict__ top_idx, const float* __restrict__ top_w,
                const uint8_t* __restrict__ dq, const uint16_t* __restrict__ dsc,
                const float* __restrict__ H, __half* __restrict__ y, __half* __restrict__ u_next,
                int* status) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ __align__(16) char dyn[];
  const int TKmax = T * k, h_ld = h + 4;
  float* hs = reinterpret_cast<float*>(dyn);  // [T*k][h+4]: H row of each (token, slot)
  uint8_t* q_s = reinterpret_cast<uint8_t*>(hs + (size_t)TKmax * h_ld);  // [N][32][h/2]
  uint16_t* sc_s = reinterpret_cast<uint16_t*>(q_s + (size_t)N * kRowsB * (h / 2));
  __shared__ float yslot[kMaxT * 8][kRowsB + 1];
  __shared__ int sel[kMaxT * 8];
  __shared__ int list[kMaxT * 8];  // pairs grouped by expert (counting sort)
  __shared__ int start[kMaxN + 1];
  const int nb = h / 32;  // q4 blocks per down row
  const int row0 = blockIdx.x * kRowsB;
  const int TK = T * k;
  if (threadIdx.x == 0) {  // pairs grouped by expert, in (token, slot) order
    int cnt[kMaxN];
    for (int e = 0; e < N; ++e) cnt[e] = 0;
    for (int x = 0; x < TK; ++x) {
      int e = top_idx[x];
      if (e < 0 || e >= N) {
        record_error(status, MOE_ERR_BOUNDS);
        e = 0;
      }
      sel[x] = e;
      ++cnt[e];
    }
    int run = 0;
    for (int e = 0; e < N; ++e) {
      start[e] = run;
      run += cnt[e];
      cnt[e] = start[e];
    }
    start[N] = run;
    for (int x = 0; x < TK; ++x) list[cnt[sel[x]]++] = x;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < TK * (h / 4); i += blockDim.x) {
    const int x = i / (h / 4), c = i - x * (h / 4);
    cp16(hs + (size_t)x * h_ld + c * 4, H + ((size_t)sel[x] * T + x / k) * h + c * 4);
  }
  for (int e = 0; e < N; ++e) {  // only the selected experts' rows are read
    if (start[e + 1] == start[e]) continue;
    const size_t row = (size_t)e * d + row0;
    stage_rows(reinterpret_cast<char*>(q_s + (size_t)e * kRowsB * (h / 2)), h / 2,
               reinterpret_cast<const char*>(dq + row * (h / 2)), h / 2, kRowsB, h / 2);
    for (int i = threadIdx.x; i < kRowsB * nb; i += blockDim.x)
      sc_s[(size_t)e * kRowsB * nb + i] = dsc[row * nb + i];
  }
  cp_wait_all();
  __syncthreads();
  // thread = (row r, quarter q): row r of the selected expert, pairs q, q+4, ...
  const int r = threadIdx.x & (kRowsB - 1), q = threadIdx.x >> 5;
  // a token selects an expert at most once, so an expert has <= T <= 32 pairs
  constexpr int kPer = kMaxT / 4;
  for (int e = 0; e < N; ++e) {
    const int ne = start[e + 1] - start[e];
    const int* le = list + start[e];
    if (ne == 0) continue;  // unselected expert: nothing read
    const uint8_t* qrow = q_s + ((size_t)e * kRowsB + r) * (h / 2);
    const uint16_t* srow = sc_s + ((size_t)e * kRowsB + r) * nb;
    float acc[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) acc[j] = 0.0f;
    for (int bb = 0; bb < nb; ++bb) {
      float w[32];
      dequant_block(qrow + bb * 16, srow[bb], w);
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int li = q + 4 * j;
        if (li < ne) {
          const float4* hc = reinterpret_cast<const float4*>(hs + (size_t)le[li] * h_ld + bb * 32);
          float a = 0.0f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 hh = hc[c];
            a = fmaf(w[4 * c], hh.x, a);
            a = fmaf(w[4 * c + 1], hh.y, a);
            a = fmaf(w[4 * c + 2], hh.z, a);
            a = fmaf(w[4 * c + 3], hh.w, a);
          }
          acc[j] += a;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int li = q + 4 * j;
      if (li < ne) yslot[le[li]][r] = acc[j];
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < T * kRowsB; x += blockDim.x) {
    const int t = x / kRowsB, rr = x - t * kRowsB;
    float acc = 0.0f;
    for (int s2 = 0; s2 < k; ++s2) acc = fmaf(top_w[t * k + s2], yslot[t * k + s2][rr], acc);
    const size_t o = (size_t)t * d + row0 + rr;
    y[o] = __float2half_rn(acc);
    if (u_next) u_next[o] = __float2half_rn(__half2float(u[o]) + acc);
  }
}

struct WsLayout {
  float* H;
  int32_t* idx;
  float* w;
  __half* ping;
  __half* pong;
  __half* y;
  size_t bytes;
};

WsLayout carve_decode(const moe_shape& s, void* base) {
  Carver c(base);
  WsLayout L;
  L.H = c.take<float>((size_t)s.N * s.T * s.h);
  L.idx = c.take<int32_t>((size_t)s.T * s.k);
  L.w = c.take<float>((size_t)s.T * s.k);
  L.ping = c.take<__half>((size_t)s.T * s.d);
  L.pong = c.take<__half>((size_t)s.T * s.d);
  L.y = c.take<__half>((size_t)s.T * s.d);
  L.bytes = c.used();
  return L;
}

size_t gateup_smem(const moe_shape& s);
size_t down_smem(const moe_shape& s);
bool decode_smem_ok(const moe_shape& s);

bool decode_shape_ok(const moe_shape* s) {
  return shape_ok(s) && s->T <= kMaxT && s->N <= kMaxN && s->k <= 8 && s->d % 32 == 0 &&
         s->d % kRowsB == 0 && s->h % kRowsA == 0 && s->h % 32 == 0 && 32 % (s->h / 32) == 0 &&
         (s->h / 32) <= 32 && decode_smem_ok(*s);
}

bool layer_ok(const moe_q4_layer* L) {
  return L && L->w_route && L->gate_qs && L->gate_scales && L->up_qs && L->up_scales &&
         L->down_qs && L->down_scales && aligned16(L->gate_qs) && aligned16(L->up_qs) &&
         aligned16(L->down_qs) && aligned16(L->w_route);
}

size_t gateup_smem(const moe_shape& s) {
  return (size_t)s.T * (s.d + 8) * 2 + (size_t)s.N * (s.d + 4) * 4 + 2 * kRowsA * (s.d / 2) +
         2 * kRowsA * (s.d / 32) * 2 + 16;
}
size_t down_smem(const moe_shape& s) {
  return (size_t)s.T * s.k * (s.h + 4) * 4 + (size_t)s.N * kRowsB * (s.h / 2) +
         (size_t)s.N * kRowsB * (s.h / 32) * 2 + 16;
}

bool decode_smem_ok(const moe_shape& s) {
  return gateup_smem(s) <= 160 * 1024 && down_smem(s) <= 160 * 1024;
}

int launch_decode_layer(const moe_shape& s, const moe_q4_layer& L, const __half* u, __half* y,
                        __half* u_next, int32_t* idx, float* w, float* H, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(decode_gateup, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             160 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(decode_down, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             160 * 1024) != cudaSuccess)
      return MOE_ERR_CUDA;
    configured[dev] = true;
  }
  MOE_PREFER_SHARED((decode_gateup));
  launch_pdl(decode_gateup, dim3(s.N * (s.h / kRowsA)), dim3(128), gateup_smem(s), st, 
      u, s.T, s.d, s.N, s.k, s.h, s.renorm, L.w_route, L.bias, L.gate_qs, L.gate_scales, L.up_qs,
      L.up_scales, H, idx, w);
  MOE_PREFER_SHARED((decode_down));
  launch_pdl(decode_down, dim3(s.d / kRowsB), dim3(128), down_smem(s), st, u, s.T, s.d, s.N, s.k, s.h, idx, w,
                                                       L.down_qs, L.down_scales, H, y, u_next,
                                                       status_word());
  return launch_status();
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_decode_workspace_bytes(const moe_shape* shape) {
  if (!moe::decode_shape_ok(shape)) return 0;
  return moe::carve_decode(*shape, nullptr).bytes;
}

extern "C" int moe_decode_layer(const moe_shape* shape, const moe_q4_layer* layer,
                                const uint16_t* u, uint16_t* y, uint16_t* u_next,
                                int32_t* top_idx, float* top_w, void* ws, size_t ws_bytes,
                                void* stream) {
  using namespace moe;
  if (!decode_shape_ok(shape) || !layer_ok(layer)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!u || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(y) || !aligned16(u_next)) return MOE_ERR_INVALID_ARG;
  WsLayout W = carve_decode(*shape, ws);
  if (!ws || ws_bytes < W.bytes) return MOE_ERR_WORKSPACE;
  return launch_decode_layer(*shape, *layer, reinterpret_cast<const __half*>(u),
                             reinterpret_cast<__half*>(y), reinterpret_cast<__half*>(u_next),
                             top_idx ? top_idx : W.idx, top_w ? top_w : W.w, W.H,
                             as_stream(stream));
}

extern "C" int moe_decode_step(const moe_shape* shape, int32_t n_layers,
                               const moe_q4_layer* layers, const uint16_t* u0, uint16_t* u_out,
                               int32_t* top_idx_all, void* ws, size_t ws_bytes, void* stream) {
  using namespace moe;
  if (!decode_shape_ok(shape) || n_layers <= 0 || !layers) return MOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!layer_ok(&layers[l])) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!u0 || !u_out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u0) || !aligned16(u_out)) return MOE_ERR_INVALID_ARG;
  WsLayout W = carve_decode(*shape, ws);
  if (!ws || ws_bytes < W.bytes) return MOE_ERR_WORKSPACE;
  const moe_shape& s = *shape;
  cudaStream_t st = as_stream(stream);
  const __half* cur = reinterpret_cast<const __half*>(u0);
  for (int l = 0; l < n_layers; ++l) {
    __half* next = l == n_layers - 1 ? reinterpret_cast<__half*>(u_out)
                                     : ((l & 1) ? W.pong : W.ping);
    int32_t* idx = top_idx_all ? top_idx_all + (size_t)l * s.T * s.k : W.idx;
    const int rc = launch_decode_layer(s, layers[l], cur, W.y, next, idx, W.w, W.H, st);
    if (rc != MOE_OK) return rc;
    cur = next;
  }
  return MOE_OK;
}
