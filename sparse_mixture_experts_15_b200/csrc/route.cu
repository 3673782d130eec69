// Router: logits z = W_route u (+ b), softmax, top-k, combine weights.
// Tutorial "Mixture of Experts MoE: how sparse activation saves compute", §3.2
// (equations z, p, a); the router runs in fp32 as its code's softmax of
// logits.float() does.
//
// Logits are a register-tiled SIMT GEMM: each thread owns 8 tokens x 8
// experts and walks the input dimension in ascending order with one fused
// multiply-add per step into a block partial, which it adds to the logit at
// each kRouteBlock boundary, so every logit follows the same blocked fp32
// order whatever the tiling (the reproducible order the routing decision
// needs).
// Top-k runs one warp per token with the logits in registers.  With at most
// 16 experts a single fused kernel (router_fused_small) does all of it.
#include <cfloat>
#include <climits>

#include "common.cuh"

namespace moe {
namespace {

// Many experts (N > 16): a block tile of 8 TG tokens x 128 experts with
// 16 TG threads, 8 x 8 logits per thread, K walked in steps of 16 through
// double-buffered shared tiles (the next step's global loads are held in
// registers while the current step computes).  Each logit's block partials
// are one thread's FMA chains, added to the logit after every 128 inputs,
// so the result equals the other router kernels bit for bit.  A thread's tokens are {4 ty + i,
// 4 TG + 4 ty + i} and its experts {4 tx + j, 64 + 4 tx + j}, so the 16-byte
// shared reads of a warp are broadcasts or consecutive.  TG (8..16) is picked
// per launch so that the tiles fill whole waves of SMs (see pick_tg).
constexpr int kBigBN = 128, kBigBK = 16;

template <typename TU, int TG>
__global__ void __launch_bounds__(16 * TG)
    router_logits_big(const TU* __restrict__ u, const float* __restrict__ w,
                      const float* __restrict__ bias, float* __restrict__ z, int T, int d, int N) {
  constexpr int BT = 8 * TG, HALF = 4 * TG, NT = 16 * TG;
  constexpr int WQ = (kBigBN * kBigBK / 4 + NT - 1) / NT;  // weight float4 loads per thread
  pdl_wait();
  pdl_allow_next();
  __shared__ __align__(16) float us[2][kBigBK][BT];
  __shared__ __align__(16) float wsm[2][kBigBK][kBigBN];
  const int t0 = blockIdx.x * BT, n0 = blockIdx.y * kBigBN;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  static_assert(kRouteBlock % kBigBK == 0, "K steps must not straddle a route block");
  // the 64 running logits of a thread live in shared memory (its own float4
  // column of acc_s [16][NT], so no synchronisation), the current block's
  // partials in registers
  extern __shared__ float4 acc_s[];
  float part[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) part[i][j] = 0.0f;
#pragma unroll
  for (int q = 0; q < 16; ++q) acc_s[q * NT + tid] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  // a K step's loads: token row tid >> 1 (8 columns at (tid & 1) * 8), and
  // 4 columns of expert row x >> 2 at (x & 3) * 4 for x = tid + q NT, q < WQ
  float ru[8];
  float4 rw[WQ];
  auto fetch = [&](int k0) {
    const int kw = min(kBigBK, d - k0);  // multiple of 8
    {
      const int lr = tid >> 1, lc = (tid & 1) * 8;
      if (t0 + lr < T && lc < kw) {
        load8(u + (size_t)(t0 + lr) * d + k0 + lc, ru);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) ru[j] = 0.0f;
      }
    }
#pragma unroll
    for (int q = 0; q < WQ; ++q) {
      const int x = tid + q * NT, lr = x >> 2, lc = (x & 3) * 4;
      rw[q] = (lr < kBigBN && n0 + lr < N && lc < kw)
                  ? *reinterpret_cast<const float4*>(w + (size_t)(n0 + lr) * d + k0 + lc)
                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
  };
  auto put = [&](int buf) {
    {
      const int lr = tid >> 1, lc = (tid & 1) * 8;
#pragma unroll
      for (int j = 0; j < 8; ++j) us[buf][lc + j][lr] = ru[j];
    }
#pragma unroll
    for (int q = 0; q < WQ; ++q) {
      const int x = tid + q * NT, lr = x >> 2, lc = (x & 3) * 4;
      if (lr < kBigBN) {
        wsm[buf][lc][lr] = rw[q].x;
        wsm[buf][lc + 1][lr] = rw[q].y;
        wsm[buf][lc + 2][lr] = rw[q].z;
        wsm[buf][lc + 3][lr] = rw[q].w;
      }
    }
  };
  fetch(0);
  put(0);
  __syncthreads();
  int buf = 0;
  // blocks of kRouteBlock inputs; inside a block the K steps run as one loop
  // (the same body for every step), the partials are added after it
  for (int kb = 0; kb < d; kb += kRouteBlock) {
    const int ke = min(kb + kRouteBlock, d);
    for (int k0 = kb; k0 < ke; k0 += kBigBK) {
      const bool more = k0 + kBigBK < d;
      if (more) fetch(k0 + kBigBK);
      // a short last step reads the zeros fetch() put past d: fma(0, 0, p)
      // leaves p unchanged, so every step runs all kBigBK columns
#pragma unroll 4
      for (int kk = 0; kk < kBigBK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(&us[buf][kk][4 * ty]);
        const float4 a1 = *reinterpret_cast<const float4*>(&us[buf][kk][HALF + 4 * ty]);
        const float4 b0 = *reinterpret_cast<const float4*>(&wsm[buf][kk][4 * tx]);
        const float4 b1 = *reinterpret_cast<const float4*>(&wsm[buf][kk][64 + 4 * tx]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; j += 2) fma2_rn(part[i][j], part[i][j + 1], b[j], b[j + 1], a[i]);
      }
      if (more) {
        put(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {  // the block ends: add its partials
      float* pq = &part[q >> 1][(q & 1) * 4];
      float4 v = acc_s[q * NT + tid];
      v.x = __fadd_rn(v.x, pq[0]);
      v.y = __fadd_rn(v.y, pq[1]);
      v.z = __fadd_rn(v.z, pq[2]);
      v.w = __fadd_rn(v.w, pq[3]);
      acc_s[q * NT + tid] = v;
      pq[0] = pq[1] = pq[2] = pq[3] = 0.0f;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? 4 * ty + i : HALF + 4 * ty + i - 4);
    if (t >= T) continue;
    const float4 v0 = acc_s[(2 * i) * NT + tid], v1 = acc_s[(2 * i + 1) * NT + tid];
    const float zi[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? 4 * tx + j : 64 + 4 * tx + j - 4);
      if (n < N) z[(size_t)t * N + n] = bias ? __fadd_rn(zi[j], bias[n]) : zi[j];
    }
  }
}

// Token-tile width 8 TG for the large router: a tile's time grows with TG
// (its FMAs), and cps[TG] tiles run at once per SM (the kernel's occupancy,
// set by its registers: 7-warp CTAs fit twice per SM only at <= 128
// registers a thread), so the step lasts about ceil(tiles / (SMs cps)) * TG;
// the least wins (larger TG on ties).  4096 tokens x 896 experts on 148
// SMs: TG = 13, 280 tiles in one wave of 2 per SM.
int pick_tg(int T, int N, int sms, const int* cps) {
  const int64_t nt = (N + kBigBN - 1) / kBigBN;
  int best = 16;
  int64_t best_cost = INT64_MAX;
  for (int tg = 16; tg >= 8; --tg) {
    const int64_t tiles = nt * ((T + 8 * tg - 1) / (8 * tg));
    const int64_t slots = (int64_t)sms * (cps[tg] > 0 ? cps[tg] : 1);
    const int64_t cost = (tiles + slots - 1) / slots * tg;
    if (cost < best_cost) {
      best_cost = cost;
      best = tg;
    }
  }
  return best;
}

// (z, index) ordering of the top-k: larger z first, equal z -> lower index.
__device__ __forceinline__ bool better(float za, int ia, float zb, int ib) {
  return za > zb || (za == zb && ia < ib);
}

template <int PER>
__global__ void __launch_bounds__(256)
    router_topk_kernel(const float* __restrict__ z, int T, int N, int k, int renorm,
                       int32_t* __restrict__ top_idx, float* __restrict__ top_w,
                       float* __restrict__ probs) {
  pdl_wait();
  pdl_allow_next();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const float* zt = z + (size_t)warp * N;
  float zr[PER];
  float zmax = -FLT_MAX;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int j = lane + 32 * q;
    zr[q] = j < N ? zt[j] : -FLT_MAX;
    zmax = fmaxf(zmax, zr[q]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
  float den = 0.0f;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int j = lane + 32 * q;
    if (j < N) den += expf(zr[q] - zmax);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (probs) {
    float* pt = probs + (size_t)warp * N;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int j = lane + 32 * q;
      if (j < N) pt[j] = expf(zr[q] - zmax) / den;
    }
  }
  uint32_t taken = 0;
  float my_z = -FLT_MAX;
  int my_i = INT_MAX;
  for (int s = 0; s < k; ++s) {
    float bz = -FLT_MAX;
    int bi = INT_MAX;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int j = lane + 32 * q;
      if (j < N && !((taken >> q) & 1u) && better(zr[q], j, bz, bi)) {
        bz = zr[q];
        bi = j;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(oz, oi, bz, bi)) {
        bz = oz;
        bi = oi;
      }
    }
    if (bi != INT_MAX && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == s) {
      my_z = bz;
      my_i = bi;
    }
  }
  const float p = lane < k ? expf(my_z - zmax) / den : 0.0f;
  float ps = p;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
  if (lane < k) {
    top_idx[(size_t)warp * k + lane] = my_i;
    top_w[(size_t)warp * k + lane] = renorm ? p / ps : p;
  }
}

// One 8-element step of a block chain: c = w[j] x[j] + c for j ascending.
template <typename TU>
__device__ __forceinline__ float dot8(float c, const TU* x, const float* w) {
  float xv[8];
  load8(x, xv);
  const float4 w0 = *reinterpret_cast<const float4*>(w);
  const float4 w1 = *reinterpret_cast<const float4*>(w + 4);
  c = __fmaf_rn(w0.x, xv[0], c);
  c = __fmaf_rn(w0.y, xv[1], c);
  c = __fmaf_rn(w0.z, xv[2], c);
  c = __fmaf_rn(w0.w, xv[3], c);
  c = __fmaf_rn(w1.x, xv[4], c);
  c = __fmaf_rn(w1.y, xv[5], c);
  c = __fmaf_rn(w1.z, xv[6], c);
  c = __fmaf_rn(w1.w, xv[7], c);
  return c;
}

// Few experts (N <= NP <= 16): a block routes 128 / NP tokens with one
// thread per (token, expert) pair, each running its logit's block chains
// over j (the same order as the tiled kernel), then one thread per
// token does softmax, top-k and the combine weights from shared memory, so
// routing is a single launch.  Per slab of inputs the block's token rows and
// the router rows are copied with cp.async (every copy issued before one
// wait) into rows padded to 16 B past a multiple of 128 B, so the 16-byte
// shared-memory reads of a warp hit distinct banks.  Optionally the block
// also writes its expert counts (the first step of the permutation).
constexpr int kRouteThreads = 128;

__device__ __forceinline__ void cp16_async(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}

template <int NP, typename TU>
__global__ void __launch_bounds__(kRouteThreads)
    router_fused_small(const TU* __restrict__ u, const float* __restrict__ w,
                       const float* __restrict__ bias, int T, int d, int N, int k, int renorm,
                       int32_t* __restrict__ top_idx, float* __restrict__ top_w,
                       float* __restrict__ probs, float* __restrict__ logits,
                       int32_t* __restrict__ hist) {
  pdl_wait();
  pdl_allow_next();
  constexpr int TPB = kRouteThreads / NP;               // tokens per block
  constexpr int kSlab = sizeof(TU) == 4 ? 128 : 256;  // 512-byte token slabs
  constexpr int kRowBytes = kSlab * (int)sizeof(TU) + 16;
  constexpr int kWld = kSlab + 4;  // padded router row (floats)
  __shared__ __align__(16) float ws[NP][kWld];
  __shared__ __align__(16) char us[TPB * kRowBytes];
  __shared__ float zs[TPB][NP + 1];
  __shared__ int cnt[NP];
  const int t0 = blockIdx.x * TPB;
  const int tl = threadIdx.x / NP, e = threadIdx.x - tl * NP;
  const int t = t0 + tl;
  float acc = 0.0f;
  for (int k0 = 0; k0 < d; k0 += kSlab) {
    const int kw = min(kSlab, d - k0);  // multiple of 8
    const int chunks = kw * (int)sizeof(TU) / 16;
    __syncthreads();
    for (int i = threadIdx.x; i < TPB * chunks; i += blockDim.x) {
      const int r = i / chunks, c = i - r * chunks;
      if (t0 + r < T)
        cp16_async(us + r * kRowBytes + c * 16,
                   reinterpret_cast<const char*>(u + (size_t)(t0 + r) * d + k0) + c * 16);
    }
    const int wchunks = kw / 4;
    for (int i = threadIdx.x; i < N * wchunks; i += blockDim.x) {
      const int ee = i / wchunks, c = i - ee * wchunks;
      cp16_async(&ws[ee][c * 4], w + (size_t)ee * d + k0 + c * 4);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (t < T && e < N) {
      const TU* ut = reinterpret_cast<const TU*>(us + tl * kRowBytes);
      const float* wt = ws[e];
      if (kSlab == 2 * kRouteBlock && kw == kSlab) {  // two blocks, chains interleaved
        float c0 = 0.0f, c1 = 0.0f;
        for (int j = 0; j < kRouteBlock; j += 8) {
          c0 = dot8(c0, ut + j, wt + j);
          c1 = dot8(c1, ut + kRouteBlock + j, wt + kRouteBlock + j);
        }
        acc = __fadd_rn(__fadd_rn(acc, c0), c1);
      } else {
        for (int jb = 0; jb < kw; jb += kRouteBlock) {
          const int je = min(jb + kRouteBlock, kw);
          float c = 0.0f;
          for (int j = jb; j < je; j += 8) c = dot8(c, ut + j, wt + j);
          acc = __fadd_rn(acc, c);
        }
      }
    }
  }
  if (e < N) {
    if (bias) acc = __fadd_rn(acc, bias[e]);
    zs[tl][e] = acc;
    if (logits && t < T) logits[(size_t)t * N + e] = acc;
  }
  if (hist && threadIdx.x < NP) cnt[threadIdx.x] = 0;
  __syncthreads();
  if (threadIdx.x < TPB && t0 + threadIdx.x < T && k == 2 && !probs) {
    // top-2 in one pass and weights from one reciprocal, as the fused
    // route+dispatch kernel does, so both give the same weights bit for bit
    const int tt = t0 + threadIdx.x;
    float zr[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) zr[i] = i < N ? zs[threadIdx.x][i] : 0.0f;
    int b0, b1;
    float z0, z1;
    top2_of<NP>(zr, N, b0, z0, b1, z1);
    const float e1 = expf(z1 - z0);
    float S = 1.0f + e1;
    if (!renorm) {
      S = 0.0f;
#pragma unroll
      for (int i = 0; i < NP; ++i)
        if (i < N) S += expf(zr[i] - z0);
    }
    const float r = 1.0f / S;
    top_idx[(size_t)tt * 2] = b0;
    top_idx[(size_t)tt * 2 + 1] = b1;
    top_w[(size_t)tt * 2] = expf(z0 - z0) * r;
    top_w[(size_t)tt * 2 + 1] = e1 * r;
    if (hist) {
      atomicAdd(&cnt[b0], 1);
      atomicAdd(&cnt[b1], 1);
    }
  } else if (threadIdx.x < TPB && t0 + threadIdx.x < T) {
    const int tt = t0 + threadIdx.x;
    const float* z = zs[threadIdx.x];
    float zmax = -FLT_MAX;
    for (int i = 0; i < N; ++i) zmax = fmaxf(zmax, z[i]);
    float den = 0.0f;
    for (int i = 0; i < N; ++i) den += expf(z[i] - zmax);
    if (probs)
      for (int i = 0; i < N; ++i) probs[(size_t)tt * N + i] = expf(z[i] - zmax) / den;
    uint32_t taken = 0;
    float psel[16];
    int isel[16];
    float ps = 0.0f;
    for (int s = 0; s < k; ++s) {
      int bi = -1;  // the running best's value kept in a register (bv == z[bi])
      float bv = 0.0f;
      for (int i = 0; i < N; ++i) {
        const float zi = z[i];
        if (!((taken >> i) & 1u) && (bi < 0 || zi > bv)) {
          bi = i;
          bv = zi;
        }
      }
      taken |= 1u << bi;
      isel[s] = bi;
      psel[s] = expf(z[bi] - zmax) / den;
      ps += psel[s];
    }
    for (int s = 0; s < k; ++s) {
      top_idx[(size_t)tt * k + s] = isel[s];
      top_w[(size_t)tt * k + s] = renorm ? psel[s] / ps : psel[s];
      if (hist) atomicAdd(&cnt[isel[s]], 1);
    }
  }
  if (hist) {  // this block's expert counts: the first step of the permutation
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x) hist[(size_t)blockIdx.x * N + i] = cnt[i];
  }
}

template <int TG>
constexpr size_t logits_smem() {
  return (size_t)64 * 4 * 16 * TG;  // acc_s: 64 fp32 logits per thread
}

// Sets the instantiation's shared-memory attributes once per device and
// returns its CTAs per SM (0 when unknown).
template <typename TU, int TG>
int logits_setup() {
  static std::atomic<bool> configured[kMaxDevices];
  static std::atomic<int> occupancy[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || !device_slot(dev)) return 0;
  if (needs_setup(configured, dev)) {
    MOE_PREFER_SHARED((router_logits_big<TU, TG>));
    cudaFuncSetAttribute(router_logits_big<TU, TG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)logits_smem<TG>());
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, router_logits_big<TU, TG>, 16 * TG,
                                                      logits_smem<TG>()) != cudaSuccess)
      n = 0;
    occupancy[dev].store(n, std::memory_order_relaxed);
    mark_setup(configured, dev);
  }
  return occupancy[dev].load(std::memory_order_relaxed);
}

template <typename TU, int TG>
void launch_logits_tg(const TU* u, const float* w, const float* bias, float* z, int T, int d,
                      int N, cudaStream_t st) {
  dim3 grid((T + 8 * TG - 1) / (8 * TG), (N + kBigBN - 1) / kBigBN);
  logits_setup<TU, TG>();
  launch_pdl(router_logits_big<TU, TG>, grid, dim3(16 * TG), logits_smem<TG>(), st, u, w, bias,
             z, T, d, N);
}

template <typename TU>
void launch_logits(const TU* u, const float* w, const float* bias, float* z, int T, int d, int N,
                   cudaStream_t st) {
  const int cps[17] = {0, 0, 0, 0, 0, 0, 0, 0,
                       logits_setup<TU, 8>(),  logits_setup<TU, 9>(),  logits_setup<TU, 10>(),
                       logits_setup<TU, 11>(), logits_setup<TU, 12>(), logits_setup<TU, 13>(),
                       logits_setup<TU, 14>(), logits_setup<TU, 15>(), logits_setup<TU, 16>()};
  switch (pick_tg(T, N, sm_count(), cps)) {
    case 8: return launch_logits_tg<TU, 8>(u, w, bias, z, T, d, N, st);
    case 9: return launch_logits_tg<TU, 9>(u, w, bias, z, T, d, N, st);
    case 10: return launch_logits_tg<TU, 10>(u, w, bias, z, T, d, N, st);
    case 11: return launch_logits_tg<TU, 11>(u, w, bias, z, T, d, N, st);
    case 12: return launch_logits_tg<TU, 12>(u, w, bias, z, T, d, N, st);
    case 13: return launch_logits_tg<TU, 13>(u, w, bias, z, T, d, N, st);
    case 14: return launch_logits_tg<TU, 14>(u, w, bias, z, T, d, N, st);
    case 15: return launch_logits_tg<TU, 15>(u, w, bias, z, T, d, N, st);
    default: return launch_logits_tg<TU, 16>(u, w, bias, z, T, d, N, st);
  }
}

}  // namespace

size_t route_ws_bytes(const moe_shape& s) { return align_up((size_t)s.T * s.N * 4, 256); }

int route_tokens_per_block(int N) { return kRouteThreads / (N <= 8 ? 8 : 16); }

int launch_route(const moe_shape& s, const void* u, int32_t u_dtype, const float* w_route,
                 const float* bias, int32_t* top_idx, float* top_w, float* probs, float* logits,
                 void* ws, cudaStream_t st, int32_t* hist) {
  if (s.T == 0) return MOE_OK;
  if (s.N <= 16) {
    const int blocks = (s.T + route_tokens_per_block(s.N) - 1) / route_tokens_per_block(s.N);
#define MOE_FUSED(NP, TU)                                                                     \
  do {                                                                                        \
    MOE_PREFER_SHARED((router_fused_small<NP, TU>));                                          \
    launch_pdl(router_fused_small<NP, TU>, dim3(blocks), dim3(kRouteThreads), 0, st,           \
               static_cast<const TU*>(u),                                                       \
                                                                w_route,                        \
                                                      bias, s.T, s.d, s.N, s.k, s.renorm,     \
                                                      top_idx, top_w, probs, logits, hist);   \
  } while (0)
    if (u_dtype == MOE_F32) {
      if (s.N <= 8) MOE_FUSED(8, float); else MOE_FUSED(16, float);
    } else if (u_dtype == MOE_BF16) {
      if (s.N <= 8) MOE_FUSED(8, __nv_bfloat16); else MOE_FUSED(16, __nv_bfloat16);
    } else {
      if (s.N <= 8) MOE_FUSED(8, __half); else MOE_FUSED(16, __half);
    }
#undef MOE_FUSED
    return launch_status();
  }
  float* z = logits ? logits : static_cast<float*>(ws);
  if (u_dtype == MOE_F32) {
    launch_logits(static_cast<const float*>(u), w_route, bias, z, s.T, s.d, s.N, st);
  } else if (u_dtype == MOE_BF16) {
    launch_logits(static_cast<const __nv_bfloat16*>(u), w_route, bias, z, s.T, s.d, s.N, st);
  } else {
    launch_logits(static_cast<const __half*>(u), w_route, bias, z, s.T, s.d, s.N, st);
  }
  const int blocks = (s.T + 7) / 8;
  const int per = (s.N + 31) / 32;
#define MOE_TOPK(P)                                                                          \
  do {                                                                                       \
    MOE_PREFER_SHARED((router_topk_kernel<P>));                                              \
    launch_pdl(router_topk_kernel<P>, dim3(blocks), dim3(256), 0, st, z, s.T, s.N, s.k, s.renorm, top_idx,       \
                                                  top_w, probs);                             \
  } while (0)
  if (per <= 1) MOE_TOPK(1);
  else if (per <= 2) MOE_TOPK(2);
  else if (per <= 4) MOE_TOPK(4);
  else if (per <= 8) MOE_TOPK(8);
  else if (per <= 16) MOE_TOPK(16);
  else MOE_TOPK(32);
#undef MOE_TOPK
  return launch_status();
}

}  // namespace moe

extern "C" size_t moe_route_workspace_bytes(const moe_shape* shape) {
  if (!moe::shape_ok(shape)) return 0;
  return moe::route_ws_bytes(*shape);
}

extern "C" int moe_route(const moe_shape* shape, const void* u, int32_t u_dtype,
                         const float* w_route, const float* bias, int32_t* top_idx, float* top_w,
                         float* probs, float* logits, void* ws, size_t ws_bytes, void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || !valid_act_dtype(u_dtype)) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!u || !w_route || !top_idx || !top_w)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(w_route)) return MOE_ERR_INVALID_ARG;
  if (!logits && shape->T > 0 && (!ws || ws_bytes < route_ws_bytes(*shape)))
    return MOE_ERR_WORKSPACE;
  return launch_route(*shape, u, u_dtype, w_route, bias, top_idx, top_w, probs, logits, ws,
                      as_stream(stream));
}
