// Routing, permutation and gather of the layer path in one cooperative launch
// (tutorial "Mixture of Experts MoE: how sparse activation saves compute",
// §3.2 router, softmax, top-k and renormalised weights; §3.5-§3.6 capacity,
// per-expert counts and grouping of the tokens by expert).
//
// CTA b owns the contiguous tokens [b tpc, (b + 1) tpc):
//   phase 1  stage its token rows and the router rows in shared memory, run
//            every (token, expert) logit in the blocked fp32 order of
//            kRouteBlock-element FMA chains (the order of the other router
//            kernels and the oracle),
//            softmax / top-k / weights with one thread per token, and count
//            its dispatches per expert -> hist[b][e].
//   barrier  (bounded, grid-wide)
//   phase 2  every CTA reads all counts: the counts of the CTAs before it are
//            its base ranks, the totals give L_e, the offsets and the
//            capacity drops (CTA 0 writes counts/offsets/overflow/totals);
//            its dispatches are ranked stably (dispatch order t k + s), so
//            the permutation equals the one of the separate kernels; every
//            kept dispatch writes row_of / perm_tok and copies its token row
//            from shared memory to the grouped rows (the gather).
// One launch replaces router + permutation + gather, with the token rows
// read from HBM once.
#include <cfloat>

#include "common.cuh"
#include "grid_sync.cuh"

namespace moe {
namespace {

constexpr int kRDThreads = 256;
constexpr int kRDMaxN = 16;
constexpr int kRDMaxGrid = 1024;
constexpr size_t kRDSmemLimit = 200 * 1024;

struct RDPlan {
  int tpc;      // tokens per CTA
  int grid;     // CTAs
  int row_bytes;
  uint32_t u, w, z, zp, sel, aw, cnt, base, len, off, wcnt, hist, total;
};

struct RDParams {
  const void* u;
  const float* w_route;
  const float* bias;
  int T, d, N, k, renorm, C;
  RDPlan plan;
  int32_t* top_idx;
  float* top_w;
  float* probs;   // nullable
  float* logits;  // nullable
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm_tok;
  int32_t* row_of;
  int32_t* overflow;
  int32_t* totals;
  void* x_rows;
  float* row_w;   // nullable: combine weight of each grouped row
  int32_t* hist;  // [grid][N] scratch
  unsigned* bar;  // [0] arrivals, [1] abort
  int* status;
};

uint32_t take(uint32_t& off, size_t bytes) {
  const uint32_t o = off;
  off += (uint32_t)((bytes + 15) / 16 * 16);
  return o;
}

bool make_rd_plan(const moe_shape& s, int32_t dtype, int sms, RDPlan* out) {
  if (s.T <= 0 || s.N > kRDMaxN || s.k > s.N || sms <= 0) return false;
  const size_t el = dtype_bytes(dtype);
  int grid = s.T < sms ? s.T : sms;
  const int tpc = (s.T + grid - 1) / grid;
  grid = (s.T + tpc - 1) / tpc;
  if (tpc * s.k > kRDThreads || grid > kRDMaxGrid) return false;
  RDPlan p{};
  p.tpc = tpc;
  p.grid = grid;
  p.row_bytes = (int)(s.d * el);
  uint32_t off = 0;
  p.u = take(off, (size_t)tpc * (p.row_bytes + 16));
  p.w = take(off, (size_t)s.N * (s.d + 4) * 4);
  p.z = take(off, (size_t)tpc * s.N * 4);
  p.zp = take(off, (size_t)((s.d + kRouteBlock - 1) / kRouteBlock) * tpc * s.N * 4);
  p.sel = take(off, (size_t)tpc * s.k * 4);
  p.aw = take(off, (size_t)tpc * s.k * 4);
  p.cnt = take(off, kRDMaxN * 4);
  p.base = take(off, kRDMaxN * 4);
  p.len = take(off, kRDMaxN * 4);
  p.off = take(off, (kRDMaxN + 1) * 4);
  p.wcnt = take(off, (kRDThreads / 32) * kRDMaxN * 4);
  p.hist = take(off, (size_t)grid * s.N * 4);
  p.total = off;
  if (off > kRDSmemLimit) return false;
  *out = p;
  return true;
}

__device__ __forceinline__ void cp16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}

template <int NP, typename TU>
__global__ void __launch_bounds__(kRDThreads, 1) route_dispatch(const __grid_constant__ RDParams p) {
  extern __shared__ __align__(16) char sm[];
  const RDPlan& P = p.plan;
  const int T = p.T, d = p.d, N = p.N, k = p.k, C = p.C;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tb = b * P.tpc;
  const int nt = min(P.tpc, T - tb);  // >= 1 by the plan
  const int ub = P.row_bytes + 16, wld = d + 4;
  char* us = sm + P.u;
  float* ws = reinterpret_cast<float*>(sm + P.w);
  float* z = reinterpret_cast<float*>(sm + P.z);
  float* zp = reinterpret_cast<float*>(sm + P.zp);
  int* sel = reinterpret_cast<int*>(sm + P.sel);
  float* aw = reinterpret_cast<float*>(sm + P.aw);
  int* cnt = reinterpret_cast<int*>(sm + P.cnt);
  int* base = reinterpret_cast<int*>(sm + P.base);
  int* len = reinterpret_cast<int*>(sm + P.len);
  int* off = reinterpret_cast<int*>(sm + P.off);
  int* wcnt = reinterpret_cast<int*>(sm + P.wcnt);
  int* hist_s = reinterpret_cast<int*>(sm + P.hist);

  // ---- phase 1: stage, route, count
  {
    const int per = P.row_bytes / 16;
    const char* src = static_cast<const char*>(p.u) + (size_t)tb * P.row_bytes;
    for (int i = tid; i < nt * per; i += blockDim.x) {
      const int r = i / per, c = i - r * per;
      cp16(us + r * ub + c * 16, src + (size_t)r * P.row_bytes + c * 16);
    }
    const int wper = d / 4;
    for (int i = tid; i < N * wper; i += blockDim.x) {
      const int r = i / wper, c = i - r * wper;
      cp16(ws + r * wld + c * 4, p.w_route + (size_t)r * d + c * 4);
    }
  }
  for (int e = tid; e < kRDMaxN; e += blockDim.x) cnt[e] = 0;
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  // block sums: unit = (token pair, expert quad, block m), whose eight
  // chains share each loaded activation (four experts) and router value (two
  // tokens); zp [m][nt][N]
  const int nblk = (d + kRouteBlock - 1) / kRouteBlock;
  {
    const int ntp = (nt + 1) / 2, neq = (N + 3) / 4, units = ntp * neq * nblk;
    for (int uu = tid; uu < units; uu += blockDim.x) {
      const int tp = uu % ntp, r = uu / ntp, eq = r % neq, m = r / neq;
      const int t0 = 2 * tp, t1 = min(t0 + 1, nt - 1), e0 = 4 * eq;
      const int j0 = m * kRouteBlock, len = min(kRouteBlock, d - j0);
      const TU* xa = reinterpret_cast<const TU*>(us + t0 * ub) + j0;
      const TU* xb = reinterpret_cast<const TU*>(us + t1 * ub) + j0;
      const float* wr[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) wr[e] = ws + min(e0 + e, N - 1) * wld + j0;
      float ca[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int j = 0; j < len; j += 8) {
        float va[8], vb[8];
        load8(xa + j, va);
        load8(xb + j, vb);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 w0 = *reinterpret_cast<const float4*>(wr[e] + j);
          const float4 w1 = *reinterpret_cast<const float4*>(wr[e] + j + 4);
          const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            ca[e] = __fmaf_rn(wv[q], va[q], ca[e]);
            cb[e] = __fmaf_rn(wv[q], vb[q], cb[e]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e0 + e < N) {
          zp[((size_t)m * nt + t0) * N + e0 + e] = ca[e];
          if (t1 != t0) zp[((size_t)m * nt + t1) * N + e0 + e] = cb[e];
        }
    }
  }
  __syncthreads();
  for (int q = tid; q < nt * N; q += blockDim.x) {
    const int tl = q / N, i = q - tl * N;
    float a = 0.0f;
    for (int m = 0; m < nblk; ++m) a = __fadd_rn(a, zp[(size_t)m * nt * N + q]);
    const float zz = p.bias ? __fadd_rn(a, p.bias[i]) : a;
    z[q] = zz;
    if (p.logits) p.logits[(size_t)(tb + tl) * N + i] = zz;
  }
  __syncthreads();
  for (int tl = tid; tl < nt; tl += blockDim.x) {
    const int t = tb + tl;
    float zr[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) zr[i] = i < N ? z[tl * N + i] : 0.0f;
    if (k == 2 && !p.probs) {
      // top-2 in one pass; e = exp(z - z_0), weights from one reciprocal
      // (renormalised: a_s = e_s / (1 + e_1); otherwise a_s = e_s / sum e)
      int b0, b1;
      float z0, z1;
      top2_of<NP>(zr, N, b0, z0, b1, z1);
      const float e1 = expf(z1 - z0);
      float S = 1.0f + e1;
      if (!p.renorm) {
        S = 0.0f;
#pragma unroll
        for (int i = 0; i < NP; ++i)
          if (i < N) S += expf(zr[i] - z0);
      }
      const float r = 1.0f / S;
      const float a0 = expf(z0 - z0) * r, a1 = e1 * r;
      sel[tl * 2] = b0;
      sel[tl * 2 + 1] = b1;
      aw[tl * 2] = a0;
      aw[tl * 2 + 1] = a1;
      p.top_idx[(size_t)t * 2] = b0;
      p.top_idx[(size_t)t * 2 + 1] = b1;
      p.top_w[(size_t)t * 2] = a0;
      p.top_w[(size_t)t * 2 + 1] = a1;
      atomicAdd(&cnt[b0], 1);
      atomicAdd(&cnt[b1], 1);
      continue;
    }
    float zmax = -FLT_MAX;
#pragma unroll
    for (int i = 0; i < NP; ++i)
      if (i < N) zmax = fmaxf(zmax, zr[i]);
    float den = 0.0f;
#pragma unroll
    for (int i = 0; i < NP; ++i)
      if (i < N) den += expf(zr[i] - zmax);
    if (p.probs)
      for (int i = 0; i < N; ++i) p.probs[(size_t)t * N + i] = expf(z[tl * N + i] - zmax) / den;
    uint32_t taken = 0;
    float psel[kRDMaxN];
    float ps = 0.0f;
    for (int s = 0; s < k; ++s) {
      int bi = -1;
      float bz = 0.0f;
#pragma unroll
      for (int i = 0; i < NP; ++i)
        if (i < N && !((taken >> i) & 1u) && (bi < 0 || zr[i] > bz)) {
          bi = i;
          bz = zr[i];
        }
      if (bi < 0) {  // only NaN logits left: the lowest free index
        bi = __ffs(~taken) - 1;
        bz = z[tl * N + bi];
      }
      taken |= 1u << bi;
      sel[tl * k + s] = bi;
      psel[s] = expf(bz - zmax) / den;
      ps += psel[s];
      atomicAdd(&cnt[bi], 1);
    }
    for (int s = 0; s < k; ++s) {
      const float a = p.renorm ? psel[s] / ps : psel[s];
      aw[tl * k + s] = a;
      p.top_idx[(size_t)t * k + s] = sel[tl * k + s];
      p.top_w[(size_t)t * k + s] = a;
    }
  }
  __syncthreads();
  for (int e = tid; e < N; e += blockDim.x) p.hist[(size_t)b * N + e] = cnt[e];
  grid_arrive(p.bar);
  if (!grid_wait(p.bar, (unsigned)gridDim.x, p.status)) return;

  // ---- phase 2: offsets, stable ranks, row_of / perm_tok, row copies
  const int G = gridDim.x, nh = G * N;
  for (int i = tid; i < nh; i += blockDim.x) hist_s[i] = __ldcg(p.hist + i);
  for (int i = tid; i < (kRDThreads / 32) * kRDMaxN; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  for (int e = warp; e < N; e += kRDThreads / 32) {  // one warp per expert
    int bs = 0, tot = 0;
    for (int i = lane; i < G; i += 32) {
      const int v = hist_s[i * N + e];
      bs += i < b ? v : 0;
      tot += v;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      bs += __shfl_xor_sync(0xffffffffu, bs, o);
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
    }
    if (lane == 0) {
      base[e] = bs;
      len[e] = tot;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0, of = 0, empty = 0;
    for (int e = 0; e < N; ++e) {
      const int L = len[e];
      off[e] = run;
      run += (C > 0 && L > C) ? C : L;
      if (C > 0 && L > C) of += L - C;
      if (C > 0 && L < C) empty += C - L;
    }
    off[N] = run;
    if (b == 0) {
      for (int e = 0; e < N; ++e) {
        p.counts[e] = len[e];
        p.offsets[e] = off[e];
        p.overflow[e] = (C > 0 && len[e] > C) ? len[e] - C : 0;
      }
      p.offsets[N] = run;
      p.totals[0] = run;
      p.totals[1] = of;
      p.totals[2] = empty;
    }
  }
  // one thread per dispatch of this CTA (nt k <= blockDim by the plan)
  const int nx = nt * k;
  const int e = tid < nx ? sel[tid] : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int in_warp = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && in_warp == 0) wcnt[warp * kRDMaxN + e] = __popc(peers);
  __syncthreads();
  int row = -1;
  if (e >= 0) {
    int cross = 0;
    for (int v = 0; v < warp; ++v) cross += wcnt[v * kRDMaxN + e];
    const int rank = base[e] + cross + in_warp;
    if (!(C > 0 && rank >= C)) row = off[e] + rank;
    const int x = tb * k + tid;
    p.row_of[x] = row;
    if (row >= 0) p.perm_tok[row] = tb + tid / k;
    if (row >= 0 && p.row_w) p.row_w[row] = aw[tid];
  }
  __syncthreads();
  // row copies: dispatch i's row into the grouped rows (one warp per dispatch)
  int* drow = reinterpret_cast<int*>(z);  // logits are no longer needed
  if (tid < nx) drow[tid] = row;
  __syncthreads();
  const int per = P.row_bytes / 16;
  for (int i = warp; i < nx; i += kRDThreads / 32) {
    const int r = drow[i];
    if (r < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(us + (i / k) * ub);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<char*>(p.x_rows) + (size_t)r * P.row_bytes);
    for (int c = lane; c < per; c += 32) dst[c] = src[c];
  }
}

}  // namespace

bool route_dispatch_ok(const moe_shape& s, int32_t dtype) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return false;
  RDPlan p;
  return (dtype == MOE_F32 || dtype == MOE_BF16) && make_rd_plan(s, dtype, sms, &p);
}

size_t route_dispatch_ws_bytes(const moe_shape& s) {
  return align_up((size_t)kRDMaxGrid * (s.N > 0 ? s.N : 1) * 4, 256) + 256;
}

int launch_route_dispatch(const moe_shape& s, const void* u, int32_t dtype, const float* w_route,
                          const float* bias, int32_t* top_idx, float* top_w, float* probs,
                          float* logits, int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                          int32_t* row_of, int32_t* overflow, int32_t* totals, void* x_rows,
                          void* ws, cudaStream_t st, float* row_w) {
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  RDParams p{};
  if (!make_rd_plan(s, dtype, sms, &p.plan)) return MOE_ERR_UNSUPPORTED;
  if (needs_setup(configured, dev)) {
    const int lim = (int)kRDSmemLimit;
    MOE_PREFER_SHARED((route_dispatch<8, float>));
    MOE_PREFER_SHARED((route_dispatch<16, float>));
    MOE_PREFER_SHARED((route_dispatch<8, __nv_bfloat16>));
    MOE_PREFER_SHARED((route_dispatch<16, __nv_bfloat16>));
    if (cudaFuncSetAttribute(route_dispatch<8, float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lim) != cudaSuccess ||
        cudaFuncSetAttribute(route_dispatch<16, float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lim) != cudaSuccess ||
        cudaFuncSetAttribute(route_dispatch<8, __nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lim) != cudaSuccess ||
        cudaFuncSetAttribute(route_dispatch<16, __nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, lim) != cudaSuccess)
      return MOE_ERR_CUDA;
    mark_setup(configured, dev);
  }
  p.u = u;
  p.w_route = w_route;
  p.bias = bias;
  p.T = s.T;
  p.d = s.d;
  p.N = s.N;
  p.k = s.k;
  p.renorm = s.renorm;
  p.C = s.capacity;
  p.top_idx = top_idx;
  p.top_w = top_w;
  p.row_w = row_w;
  p.probs = probs;
  p.logits = logits;
  p.counts = counts;
  p.offsets = offsets;
  p.perm_tok = perm_tok;
  p.row_of = row_of;
  p.overflow = overflow;
  p.totals = totals;
  p.x_rows = x_rows;
  p.hist = static_cast<int32_t*>(ws);
  p.bar = reinterpret_cast<unsigned*>(static_cast<char*>(ws) +
                                      align_up((size_t)kRDMaxGrid * s.N * 4, 256));
  p.status = status_word();
  if (cudaMemsetAsync(p.bar, 0, 4 * sizeof(unsigned), st) != cudaSuccess) return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.plan.grid);
  cfg.blockDim = dim3(kRDThreads);
  cfg.dynamicSmemBytes = p.plan.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (dtype == MOE_F32)
    e = s.N <= 8 ? cudaLaunchKernelEx(&cfg, route_dispatch<8, float>, p)
                 : cudaLaunchKernelEx(&cfg, route_dispatch<16, float>, p);
  else
    e = s.N <= 8 ? cudaLaunchKernelEx(&cfg, route_dispatch<8, __nv_bfloat16>, p)
                 : cudaLaunchKernelEx(&cfg, route_dispatch<16, __nv_bfloat16>, p);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
