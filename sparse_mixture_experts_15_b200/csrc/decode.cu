// Small-batch decode path with q4_0 experts.
//
// Deployment notes "Kestrel-MCU notes 13", §2 and §4: per layer the router
// GEMV picks the top-k experts, and only the selected experts' gate/up/down
// weights are read ("lookup loading"), stored as q4_0 (32-value blocks, one
// fp16 scale s, 4-bit q, w = (q - 8) s).  The tutorial "Mixture of Experts
// MoE: how sparse activation saves compute" §3.1-§3.2 fixes the arithmetic.
// Layers chain as u_{l+1} = fp16(u_l + y_l).
//
// At decode sizes a layer moves well under a megabyte, so the step is bound
// by its chain of dependent phases, not by HBM.  All layers of a call run in
// ONE persistent cooperative launch (at most one CTA per SM, all
// co-resident).  Two kernels: the one-barrier kernel (further below: items
// of (token, slot, hidden slice), one grid barrier per layer) when its
// shared-memory plan fits, else the two-phase kernel described here, with
// two grid barriers per layer instead of two kernel boundaries:
//   route   every CTA stages u_l and W_route (fp32) in shared memory and
//           routes all T tokens itself (identical, deterministic code, so
//           every CTA holds the same selection); the pairs are grouped by
//           expert.  (The next layer's router rows are fetched while the
//           CTA waits at the first barrier.)
//   phase A items (selected expert, RA hidden rows) are spread over the
//           CTAs: the item's gate/up q4 rows are staged in shared memory
//           and dequantised in registers inside the (row, token) dots;
//           H[e][t][rows] = SiLU(g) * v goes to global memory (L2).
//   barrier
//   phase B units of (one token, RB output rows), T * d / RB of them: the
//           token's k selected experts' down rows of the unit were staged
//           before the barrier; each slot's H row (read from L2) is dotted
//           with them, the slots are summed in order,
//           y = sum_s a_s W_down H, u_{l+1} = fp16(u_l + y).  A unit reads
//           only its token's k rows of H, so an H row is read by d / RB CTAs
//           rather than by every CTA.
//   barrier
// Unselected experts' weights are never read.  Every barrier wait is bounded
// (2 s of device time); on timeout the kernel records MOE_ERR_TIMEOUT, raises
// an abort flag that releases every other CTA, and all CTAs return.
#include <cfloat>

#include "common.cuh"
#include "grid_sync.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxT = 32;            // decode batch limit
constexpr int kMaxN = 64;            // expert limit (64-bit selection mask)
constexpr int kLayersPerLaunch = 32; // layer descriptors carried by one launch
constexpr size_t kSmemLimit = 226 * 1024;  // dynamic; leaves room for static

__device__ __forceinline__ float f16f(uint16_t c) { return __half2float(__ushort_as_half(c)); }

// q - 8 as fp32 for the 4 nibbles (each 0..15) held in the bytes of v:
// the bytes are placed under the exponent of 2^23, so the float is 2^23 + q
// exactly, and subtracting 2^23 + 8 is exact too (no int-to-float convert).
__device__ __forceinline__ float nib(uint32_t v, int b) {
  return __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7540 | b)) - 8388616.0f;
}

// Sum over one q4_0 block of (q - 8) x (byte j of the block holds element j
// in its low nibble and element j + 16 in its high one): four chains, added
// pairwise; the caller applies the block scale once.
__device__ __forceinline__ float q4_block_dot(const uint8_t* qs, const float* x) {
  const uint4 raw = *reinterpret_cast<const uint4*>(qs);
  const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = wd[i] & 0x0F0F0F0Fu, hi = (wd[i] >> 4) & 0x0F0F0F0Fu;
    a0 = fmaf(nib(lo, 0), x[4 * i], a0);
    a1 = fmaf(nib(lo, 1), x[4 * i + 1], a1);
    a2 = fmaf(nib(lo, 2), x[4 * i + 2], a2);
    a3 = fmaf(nib(lo, 3), x[4 * i + 3], a3);
    a0 = fmaf(nib(hi, 0), x[16 + 4 * i], a0);
    a1 = fmaf(nib(hi, 1), x[16 + 4 * i + 1], a1);
    a2 = fmaf(nib(hi, 2), x[16 + 4 * i + 2], a2);
    a3 = fmaf(nib(hi, 3), x[16 + 4 * i + 3], a3);
  }
  return (a0 + a1) + (a2 + a3);
}


// Asynchronous global -> shared copies (LDGSTS), all issued before one wait.
// The .cg form reads through L2 only, so data written by other CTAs of this
// launch before a grid barrier is seen.
__device__ __forceinline__ void cp16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem))),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// cp.async groups: the copies issued since the last commit form one group;
// wait_group<n> returns once at most n of this thread's groups are pending.
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// rows x row_bytes (multiple of 16) from gmem (row stride g_stride bytes) to
// shared rows of s_stride bytes; all threads of the CTA cooperate.
__device__ __forceinline__ void stage_rows(char* smem, int s_stride, const char* gmem,
                                           size_t g_stride, int rows, int row_bytes) {
  const int per_row = row_bytes / 16;
  if (per_row <= (int)blockDim.x && blockDim.x % per_row == 0) {
    // a thread keeps one 16-byte column and walks the rows: no division per copy
    const int c = threadIdx.x % per_row, step = blockDim.x / per_row;
    for (int r = threadIdx.x / per_row; r < rows; r += step)
      cp16(smem + (size_t)r * s_stride + c * 16, gmem + r * g_stride + (size_t)c * 16);
    return;
  }
  for (int i = threadIdx.x; i < rows * per_row; i += blockDim.x) {
    const int r = i / per_row, c = i - r * per_row;
    cp16(smem + (size_t)r * s_stride + c * 16, gmem + r * g_stride + (size_t)c * 16);
  }
}

// A contiguous byte range (both ends 4-byte aligned) to shared memory, in
// 16-byte copies when both addresses and the size allow it.
__device__ __forceinline__ void stage_bytes(void* smem, const void* gmem, int nbytes) {
  char* s = static_cast<char*>(smem);
  const char* g = static_cast<const char*>(gmem);
  if (((reinterpret_cast<uintptr_t>(s) | reinterpret_cast<uintptr_t>(g) | (uintptr_t)nbytes) &
       15u) == 0) {
    for (int i = threadIdx.x; i < nbytes / 16; i += blockDim.x) cp16(s + 16 * i, g + 16 * i);
  } else {
    for (int i = threadIdx.x; i < nbytes / 4; i += blockDim.x) cp4(s + 4 * i, g + 4 * i);
  }
}

// Softmax and top-k of one token for N up to 64, logits read from shared
// memory (the register version above covers N <= 32).
__device__ __noinline__ void topk_wide(const float* zt, int N, int k, int renorm, int* sel,
                                       float* aw) {
  float zmax = -FLT_MAX;
  for (int i = 0; i < N; ++i) zmax = fmaxf(zmax, zt[i]);
  float den = 0.0f;
  for (int i = 0; i < N; ++i) den += expf(zt[i] - zmax);
  uint64_t taken = 0;
  float ps = 0.0f;
  float a[8];
  for (int s = 0; s < k; ++s) {
    // the running best kept in a register (bv == zt[bi]), so no comparison
    // waits on a load whose address depends on the previous one
    int bi = -1;
    float bv = 0.0f;
    for (int i = 0; i < N; ++i) {
      const float zi = zt[i];
      if (!((taken >> i) & 1ull) && (bi < 0 || zi > bv)) {
        bi = i;
        bv = zi;
      }
    }
    if (bi < 0) bi = __ffsll((long long)~taken) - 1;  // only NaN logits left
    taken |= 1ull << bi;
    sel[s] = bi;
    a[s] = expf(zt[bi] - zmax) / den;
    ps += a[s];
  }
  for (int s = 0; s < k; ++s) aw[s] = renorm ? a[s] / ps : a[s];
}

// Softmax, top-k and combine weights of one token from its N logits zt
// (N <= NR).  The k largest logits in descending order, ties to the lower
// index (the selection loop of the other router kernels).  With z_0 the
// first selected logit (the largest) and e_i = exp(z_i - z_0): renormalised
// weights a_s = e_s / sum of the selected e (e_0 = 1), otherwise a_s = e_s /
// sum of all N e_i.  One reciprocal replaces the per-slot divisions, and the
// slot loop is unrolled so the slots stay in registers: this code runs once
// per layer on the critical path, where a dependent division costs about 90
// cycles and a loop branch about 20.
template <int NR>
__device__ __forceinline__ void topk_token(const float* zt, int N, int k, int renorm, int* sel,
                                           float* aw) {
  float zr[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) zr[i] = i < N ? zt[i] : 0.0f;
  uint32_t taken = 0;
  int si[8];
  float zs[8];
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    if (s < k) {
      int bi = -1;
      float bz = 0.0f;
#pragma unroll
      for (int i = 0; i < NR; ++i)
        if (i < N && !((taken >> i) & 1u) && (bi < 0 || zr[i] > bz)) {
          bi = i;
          bz = zr[i];
        }
      if (bi < 0) {  // only NaN logits left: take the lowest free index
        bi = __ffs(~taken) - 1;
#pragma unroll
        for (int i = 0; i < NR; ++i)
          if (i == bi) bz = zr[i];
      }
      taken |= 1u << bi;
      si[s] = bi;
      zs[s] = bz;
    }
  }
  const float z0 = zs[0];
  float e[8], S = 0.0f;
#pragma unroll
  for (int s = 0; s < 8; ++s)
    if (s < k) {
      e[s] = expf(zs[s] - z0);
      S += e[s];
    }
  if (!renorm) {
    S = 0.0f;
#pragma unroll
    for (int i = 0; i < NR; ++i)
      if (i < N) S += expf(zr[i] - z0);
  }
  const float r = 1.0f / S;
#pragma unroll
  for (int s = 0; s < 8; ++s)
    if (s < k) {
      sel[s] = si[s];
      aw[s] = e[s] * r;
    }
}

// The same selection and weights for N = 8 experts, top-2 (the common decode
// shape), with the logits in registers: one pass keeps the best two in the
// order of the selection loop (larger z first, ties to the lower index, and
// a NaN held only where that loop would hold it).
__device__ __forceinline__ void topk8_k2(const float* zt, int renorm, int* sel, float* aw) {
  const float4 za = *reinterpret_cast<const float4*>(zt);
  const float4 zb = *reinterpret_cast<const float4*>(zt + 4);
  const float zr[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
  int b0, b1;
  float z0, z1;
  top2_of<8>(zr, 8, b0, z0, b1, z1);
  const float e1 = expf(z1 - z0);
  float S = 1.0f + e1;
  if (!renorm) {
    S = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) S += expf(zr[i] - z0);
  }
  const float r = 1.0f / S;
  sel[0] = b0;
  sel[1] = b1;
  aw[0] = expf(z0 - z0) * r;
  aw[1] = e1 * r;
}

// Block sums of the router logits: unit (token t, block m, expert group g of
// E) runs the group's E chains over the block's kRouteBlock inputs, with the
// next 8 inputs' shared-memory operands loaded while the current 8 FMAs of
// each chain run.  The units of a warp are consecutive tokens of one (m, g),
// so router-row reads are broadcasts and activation reads (rows padded 16 B
// past a multiple of 128 B) hit distinct banks.  Results go to zp [m][N][T].
template <int E>
__device__ __forceinline__ void route_chains(const __half* u_s, int us_ld, const float* w_s,
                                             int ws_ld, int T, int d, int N, float* zp) {
  const int nblk = (d + kRouteBlock - 1) / kRouteBlock, ng = (N + E - 1) / E;
  const int units = T * ng * nblk;
  for (int uu = threadIdx.x; uu < units; uu += blockDim.x) {
    const int t = uu % T, r = uu / T, g = r % ng, m = r / ng;
    const int j0 = m * kRouteBlock, steps = min(kRouteBlock, d - j0) / 8;
    const int e0 = E * g, nv = min(E, N - e0);
    const uint4* ut = reinterpret_cast<const uint4*>(u_s + (size_t)t * us_ld + j0);
    const float4* wr[E];
#pragma unroll
    for (int e = 0; e < E; ++e)
      wr[e] = reinterpret_cast<const float4*>(w_s + (size_t)(e0 + min(e, nv - 1)) * ws_ld + j0);
    float c[E];
    float4 wa[E], wb[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      c[e] = 0.0f;
      wa[e] = wr[e][0];
      wb[e] = wr[e][1];
    }
    uint4 xu = ut[0];
    for (int st = 0; st < steps; ++st) {
      const int sn = st + 1 < steps ? st + 1 : st;  // the next step (a repeat at the end)
      const uint4 nxu = ut[sn];
      float4 na[E], nb[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        na[e] = wr[e][2 * sn];
        nb[e] = wr[e][2 * sn + 1];
      }
      const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w};
      float x[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&xw[q]));
        x[2 * q] = f.x;
        x[2 * q + 1] = f.y;
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        c[e] = __fmaf_rn(wa[e].x, x[0], c[e]);
        c[e] = __fmaf_rn(wa[e].y, x[1], c[e]);
        c[e] = __fmaf_rn(wa[e].z, x[2], c[e]);
        c[e] = __fmaf_rn(wa[e].w, x[3], c[e]);
        c[e] = __fmaf_rn(wb[e].x, x[4], c[e]);
        c[e] = __fmaf_rn(wb[e].y, x[5], c[e]);
        c[e] = __fmaf_rn(wb[e].z, x[6], c[e]);
        c[e] = __fmaf_rn(wb[e].w, x[7], c[e]);
        wa[e] = na[e];
        wb[e] = nb[e];
      }
      xu = nxu;
    }
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (e < nv) zp[((size_t)m * N + e0 + e) * T + t] = c[e];
  }
}

// Routing of all T tokens inside one CTA from u_s [T] rows (fp16, row stride
// us_ld elements) and w_s [N] rows (fp32, stride ws_ld), both in shared
// memory.  The logits follow the blocked order of kRouteBlock-element
// chains: the block sums come from route_chains, with the smallest expert
// group E that still gives every thread at most one unit (fewer chains per
// thread, shorter dependent work), then each logit adds its blocks in
// ascending order.  When zb_g is given, the block sums were already formed
// by the previous layer's phase B (global [nblk][N][T], read through L2) and
// neither u_s nor w_s is read.  Ties go to the lower expert index.  Leaves
// sel[t][s] and aw[t][s] in shared memory.
__device__ void route_in_cta(const __half* u_s, int us_ld, const float* w_s, int ws_ld, int T,
                             int d, int N, int k, int renorm, const float* __restrict__ bias,
                             float* z, float* zp, const float* zb_g, int* sel, float* aw) {
  const int nblk = (d + kRouteBlock - 1) / kRouteBlock, nt = blockDim.x;
  if (!zb_g) {
    if (T * N * nblk <= nt)
      route_chains<1>(u_s, us_ld, w_s, ws_ld, T, d, N, zp);
    else if (T * ((N + 1) / 2) * nblk <= nt)
      route_chains<2>(u_s, us_ld, w_s, ws_ld, T, d, N, zp);
    else
      route_chains<4>(u_s, us_ld, w_s, ws_ld, T, d, N, zp);
    __syncthreads();
  }
  for (int q = threadIdx.x; q < T * N; q += blockDim.x) {
    const int i = q / T, t = q - i * T;
    float zz = 0.0f;
    if (zb_g)
      for (int m = 0; m < nblk; ++m) zz = __fadd_rn(zz, __ldcg(zb_g + ((size_t)m * N + i) * T + t));
    else
      for (int m = 0; m < nblk; ++m) zz = __fadd_rn(zz, zp[((size_t)m * N + i) * T + t]);
    z[t * N + i] = bias ? __fadd_rn(zz, bias[i]) : zz;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    if (N == 8 && k == 2)
      topk8_k2(z + t * N, renorm, sel + t * k, aw + t * k);
    else if (N <= 8)
      topk_token<8>(z + t * N, N, k, renorm, sel + t * k, aw + t * k);
    else if (N <= 32)
      topk_token<32>(z + t * N, N, k, renorm, sel + t * k, aw + t * k);
    else
      topk_wide(z + t * N, N, k, renorm, sel + t * k, aw + t * k);
  }
  __syncthreads();
}

// ------------------------------------------------------------ launch plan
struct LayerPtrs {
  const float* w_route;
  const float* bias;
  const uint8_t* gq;
  const uint16_t* gs;
  const uint8_t* uq;
  const uint16_t* us;
  const uint8_t* dq;
  const uint16_t* ds;
};

// Shared-memory layout (byte offsets) and work split of one launch.
struct Plan {
  int RA;        // hidden rows per phase-A item (gate and up each)
  int RB;        // output rows per phase-B unit (one token x RB rows)
  int nbuf;      // router-weight buffers (2: next layer prefetched)
  int nsel_max;  // experts a layer can select: min(N, T*k)
  int part_cap;  // floats of the phase-A partial-sum buffer
  int early;     // 1: phase B forms the next layer's router block sums (RB a
                 // multiple of kRouteBlock, next router rows prefetched)
  uint32_t u, wr0, wr1, z, sel, aw, cnt, start, fill, list, esel, epos, misc;
  uint32_t aq, as, part, bq, bs, zs;
  uint32_t total;
};

struct Params {
  LayerPtrs layer[kLayersPerLaunch];
  int n_layers;
  int T, d, N, k, h, renorm;
  Plan plan;
  const __half* u_in;   // layer 0 input
  __half* u_work;       // inputs of layers 1.. (updated in place)
  __half* u_out;        // last layer's u_next (nullable)
  __half* y;            // last layer's y (nullable)
  int32_t* top_idx;     // [n_layers][T][k] (nullable)
  float* top_w;         // [T][k] of the last layer (nullable)
  float* H;             // [N][T][h] fp32 scratch
  float* zb;            // [d / kRouteBlock][N][T] next layer's router block sums
  unsigned* bar;        // [0] arrivals, [1] abort
  int* status;
  unsigned long long* stamps;  // nullable: [n_layers][kStamps] SM cycle stamps of CTA 0
};

// Phase boundaries stamped per layer when a trace buffer is given: 0 layer
// start, 1 input staged, 2 routed, 3 pairs grouped, 4 gate/up rows staged,
// 5 dequantised, 6 dots formed, 7 phase A done (H stored), 8 first barrier
// passed, 9 down rows ready, 10 down dots formed, 11 phase B done (u_next
// stored), 12 second barrier passed.  Stamps 4-6 and 9-10 are block 0's
// first item / slice (taken at 7 and 11 when it has none).
constexpr int kStamps = 13;

__device__ __forceinline__ void stamp(const Params& p, int l, int i) {
  if (p.stamps && blockIdx.x == 0 && threadIdx.x == 0)
    p.stamps[(size_t)l * kStamps + i] = clock64();
}

uint32_t take(uint32_t& off, size_t bytes) {
  const uint32_t o = off;
  off += (uint32_t)((bytes + 15) / 16 * 16);
  return o;
}

bool make_plan(const moe_shape& s, int sms, Plan* out) {
  const int T = s.T, d = s.d, N = s.N, k = s.k, h = s.h;
  const int nb = d / 32, nbh = h / 32;
  // phase-B units are (token, RB output rows): ideally the T * d / RB units
  // fill at most one wave of CTAs, and each unit reads only its token's k
  // rows of H; RB divides d.  Of the plans that fit shared memory (RB, then
  // the router buffers, then RA descending), the one with the fewest phase-A
  // items plus phase-B units per CTA wins, a plan without routing from the
  // previous layer's block sums counting two more (a CTA runs its items and
  // units one after another, each a staging round trip and its dots); ties
  // keep the earlier plan.
  int RB_max = 4;
  while (RB_max < d && d % (2 * RB_max) == 0 && (int64_t)T * (d / RB_max) > sms) RB_max *= 2;
  const int nsel_max = N < T * k ? N : T * k;
  bool found = false;
  int best = 0;
  for (int RB = RB_max; RB >= 4; RB /= 2)
  for (int nbuf = 2; nbuf >= 1; --nbuf) {
    for (int RA = 8; RA >= 2; RA /= 2) {
      Plan p{};
      p.RA = RA;
      p.RB = RB;
      p.nbuf = nbuf;
      p.nsel_max = nsel_max;
      // >= 2 (g, v) x units x 2 tokens; the routing's block sums share it
      p.part_cap = 2048 + 4 * RA * T;
      const int route_parts = T * N * ((d + kRouteBlock - 1) / kRouteBlock);
      if (p.part_cap < route_parts) p.part_cap = route_parts;
      if (p.part_cap < RB) p.part_cap = RB;  // phase B's u_next rows (fp32)
      p.early = nbuf == 2 && RB % kRouteBlock == 0 && d % kRouteBlock == 0;
      uint32_t off = 0;
      p.u = take(off, (size_t)T * (d + 8) * 2);
      p.wr0 = take(off, (size_t)N * (d + 4) * 4);
      p.wr1 = nbuf == 2 ? take(off, (size_t)N * (d + 4) * 4) : p.wr0;
      p.z = take(off, (size_t)T * N * 4);
      p.sel = take(off, (size_t)T * k * 4);
      p.aw = take(off, (size_t)T * k * 4);
      p.cnt = take(off, (size_t)N * 4);
      p.start = take(off, (size_t)(N + 1) * 4);
      p.fill = take(off, (size_t)N * 4);
      p.list = take(off, (size_t)T * k * 4);
      p.esel = take(off, (size_t)N * 4);
      p.epos = take(off, (size_t)N * 4);
      p.misc = take(off, 16);
      p.aq = take(off, (size_t)2 * RA * (d / 2));
      p.as = take(off, (size_t)2 * RA * nb * 2);
      p.part = take(off, (size_t)p.part_cap * 4);
      p.bq = take(off, (size_t)k * RB * (h / 2));
      p.bs = take(off, (size_t)k * RB * nbh * 2);
      p.zs = take(off, (size_t)k * (RB + 1) * 4);
      p.total = off;
      if (off > kSmemLimit) continue;
      const int items = nsel_max * (h / RA), units = T * (d / RB);
      int grid = items > units ? items : units;
      if (grid > sms) grid = sms;
      if (grid < 1) grid = 1;  // T = 0: no items and no units
      const int score = (items + grid - 1) / grid + (units + grid - 1) / grid + (p.early ? 0 : 2);
      if (!found || score < best) {
        *out = p;
        best = score;
        found = true;
      }
    }
  }
  return found;
}

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1) decode_persistent(const __grid_constant__ Params p) {
  extern __shared__ __align__(16) char sm[];
  const Plan& P = p.plan;
  const int T = p.T, d = p.d, N = p.N, k = p.k, h = p.h, Tk = T * k;
  const int RA = P.RA, RB = P.RB, nb = d / 32, nbh = h / 32;
  const int us_ld = d + 8, ws_ld = d + 4;
  const int G = gridDim.x, b = blockIdx.x, tid = threadIdx.x;
  __half* u_s = reinterpret_cast<__half*>(sm + P.u);
  float* z = reinterpret_cast<float*>(sm + P.z);
  int* sel = reinterpret_cast<int*>(sm + P.sel);
  float* aw = reinterpret_cast<float*>(sm + P.aw);
  int* cnt = reinterpret_cast<int*>(sm + P.cnt);
  int* start = reinterpret_cast<int*>(sm + P.start);
  int* fill = reinterpret_cast<int*>(sm + P.fill);
  int* list = reinterpret_cast<int*>(sm + P.list);
  int* esel = reinterpret_cast<int*>(sm + P.esel);
  int* epos = reinterpret_cast<int*>(sm + P.epos);
  int* nsel_s = reinterpret_cast<int*>(sm + P.misc);
  uint8_t* aq = reinterpret_cast<uint8_t*>(sm + P.aq);
  uint16_t* as = reinterpret_cast<uint16_t*>(sm + P.as);
  float* part = reinterpret_cast<float*>(sm + P.part);
  uint8_t* bq = reinterpret_cast<uint8_t*>(sm + P.bq);
  uint16_t* bs = reinterpret_cast<uint16_t*>(sm + P.bs);
  float* zs = reinterpret_cast<float*>(sm + P.zs);
  const int slicesA = h / RA, nsl = d / RB, nunits = T * nsl;
  unsigned n_bar = 0;

  stage_rows(sm + P.wr0, ws_ld * 4, reinterpret_cast<const char*>(p.layer[0].w_route),
             (size_t)d * 4, N, d * 4);
  // Block b's phase-A item of the next layer is staged during the first
  // barrier when every expert is likely to be selected (T k >= N): with all
  // N experts selected, block b's item is expert b / slicesA, slice
  // b % slicesA.  `spec` says that aq / as hold that item for layer l.
  bool spec = false;
  for (int l = 0; l < p.n_layers; ++l) {
    const LayerPtrs& L = p.layer[l];
    const bool last = l == p.n_layers - 1;
    const __half* u_cur = l == 0 ? p.u_in : p.u_work;
    __half* u_next = last ? p.u_out : p.u_work;
    stamp(p, l, 0);
    float* wr_s = reinterpret_cast<float*>(sm + ((l & 1) && P.nbuf == 2 ? P.wr1 : P.wr0));
    if (l > 0 && P.nbuf == 1)
      stage_rows(reinterpret_cast<char*>(wr_s), ws_ld * 4,
                 reinterpret_cast<const char*>(L.w_route), (size_t)d * 4, N, d * 4);
    stage_rows(reinterpret_cast<char*>(u_s), us_ld * 2, reinterpret_cast<const char*>(u_cur),
               (size_t)d * 2, T, d * 2);
    for (int e = tid; e < N; e += blockDim.x) cnt[e] = 0;
    // ---- routing (every CTA), then the pairs grouped by expert.  With the
    // block sums formed by the previous layer's phase B, routing runs while
    // u_l is still being staged (and stamps 1 and 2 both follow it).
    const bool early = P.early && l > 0;
    if (early) {
      __syncthreads();
      route_in_cta(u_s, us_ld, wr_s, ws_ld, T, d, N, k, p.renorm, L.bias, z, part, p.zb, sel, aw);
      cp_wait_all();
      __syncthreads();
      stamp(p, l, 1);
    } else {
      cp_wait_all();
      __syncthreads();
      stamp(p, l, 1);
      route_in_cta(u_s, us_ld, wr_s, ws_ld, T, d, N, k, p.renorm, L.bias, z, part, nullptr, sel,
                   aw);
    }
    stamp(p, l, 2);
    if (b == 0) {
      for (int x = tid; x < Tk; x += blockDim.x) {
        if (p.top_idx) p.top_idx[(size_t)l * Tk + x] = sel[x];
        if (last && p.top_w) p.top_w[x] = aw[x];
      }
    }
    // counts by shared atomics, starts and the selected-expert list by one
    // warp (N <= 64: two experts per lane), then each pair's token is placed
    // in its expert's list.  The order inside a list does not affect any
    // result (every (row, token) dot is formed the same way).
    for (int x = tid; x < Tk; x += blockDim.x) atomicAdd(&cnt[sel[x]], 1);
    __syncthreads();
    if (tid < 32) {
      const int lane = tid;
      const int c0 = lane < N ? cnt[lane] : 0, c1 = lane + 32 < N ? cnt[lane + 32] : 0;
      int s0 = c0, s1 = c1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v0 = __shfl_up_sync(0xffffffffu, s0, o), v1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
          s0 += v0;
          s1 += v1;
        }
      }
      const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
      const unsigned f0 = __ballot_sync(0xffffffffu, c0 > 0), f1 = __ballot_sync(0xffffffffu, c1 > 0);
      const unsigned lt = (1u << lane) - 1u;
      if (lane < N) {
        start[lane] = s0 - c0;
        fill[lane] = s0 - c0;
        const int r = __popc(f0 & lt);
        epos[lane] = c0 ? r : -1;
        if (c0) esel[r] = lane;
      }
      if (lane + 32 < N) {
        start[lane + 32] = tot0 + s1 - c1;
        fill[lane + 32] = tot0 + s1 - c1;
        const int r = __popc(f0) + __popc(f1 & lt);
        epos[lane + 32] = c1 ? r : -1;
        if (c1) esel[r] = lane + 32;
      }
      if (lane == 0) {
        start[N] = Tk;
        *nsel_s = __popc(f0) + __popc(f1);
      }
    }
    __syncthreads();
    for (int x = tid; x < Tk; x += blockDim.x) list[atomicAdd(&fill[sel[x]], 1)] = x / k;
    const int nsel = *nsel_s;

    // ---- issue this CTA's first phase-A item and the down rows of its first
    // phase-B slice together, before the first wait.
    const int nitems = nsel * slicesA;
    auto stage_rows_of = [&](const LayerPtrs& Lx, int e, int sl) {
      const size_t row = (size_t)e * h + (size_t)sl * RA;
      stage_bytes(aq, Lx.gq + row * (d / 2), RA * (d / 2));
      stage_bytes(aq + RA * (d / 2), Lx.uq + row * (d / 2), RA * (d / 2));
      stage_bytes(as, Lx.gs + row * nb, RA * nb * 2);
      stage_bytes(as + RA * nb, Lx.us + row * nb, RA * nb * 2);
    };
    auto stage_item = [&](int it) { stage_rows_of(L, esel[it / slicesA], it % slicesA); };
    // the down rows of phase-B unit un (token un / nsl, rows (un % nsl) RB..)
    // of the token's k selected experts, slot s at bq + s RB h/2
    auto stage_unit = [&](int un) {
      const int t = un / nsl, sl = un - t * nsl;
      for (int s2 = 0; s2 < k; ++s2) {
        const size_t row = (size_t)sel[t * k + s2] * d + (size_t)sl * RB;
        stage_bytes(bq + (size_t)s2 * RB * (h / 2), L.dq + row * (h / 2), RB * (h / 2));
        stage_bytes(bs + (size_t)s2 * RB * nbh, L.ds + row * nbh, RB * nbh * 2);
      }
    };
    __syncthreads();  // list complete before the item loop reads it
    stamp(p, l, 3);
    // Separate cp.async groups: phase A waits for its gate/up rows only, not
    // for the down rows of the phase-B unit (needed after the barrier).
    // (the speculative rows are already there when block b's item is the
    // predicted one: experts 0 .. b / slicesA all selected)
    if (b < nitems && !(spec && esel[b / slicesA] == b / slicesA)) stage_item(b);
    cp_commit();
    if (b < nunits) stage_unit(b);
    cp_commit();
    // ---- phase A: H[e][t][rows] = SiLU(W_gate u) * (W_up u) for the items
    for (int it = b; it < nitems; it += G) {
      const int e = esel[it / slicesA], sl = it % slicesA;
      const int ne = start[e + 1] - start[e];
      const int* toks = list + start[e];
      if (it != b) {
        stage_item(it);
        cp_commit();
        cp_wait_group<0>();
      } else {
        cp_wait_group<1>();  // this item's group; the slice's may still be in flight
      }
      __syncthreads();
      if (it == b) {  // (the weights are dequantised in registers inside the dots)
        stamp(p, l, 4);
        stamp(p, l, 5);
      }
      // unit = (token pair, hidden row r, part of d): one thread forms the
      // gate and the up dot of row r for two tokens, so each weight and
      // activation it loads feeds two FMAs.  d is split into nparts so that
      // about a CTA's worth of units run at once.
      const int npairs = (ne + 1) >> 1;
      int nparts = 1;
      while (nparts < nb && npairs * RA * nparts < kThreads) nparts *= 2;
      const int units = nparts * RA * npairs;
      for (int uu = tid; uu < units; uu += blockDim.x) {
        const int ip = uu % npairs, rest = uu / npairs;
        const int r = rest % RA, pp = rest / RA;
        const int i0 = 2 * ip, i1 = i0 + 1 < ne ? i0 + 1 : i0;
        const int b0 = pp * nb / nparts, b1 = (pp + 1) * nb / nparts;
        // q4_0 rows r of gate and up: nibbles and block scales staged in
        // shared memory, dequantised in registers 8 elements at a time
        const uint8_t* gq_r = aq + (size_t)r * (d / 2);
        const uint8_t* vq_r = aq + (size_t)(RA + r) * (d / 2);
        const uint16_t* gs_r = as + (size_t)r * nb;
        const uint16_t* vs_r = as + (size_t)(RA + r) * nb;
        const uint4* x0r = reinterpret_cast<const uint4*>(u_s + (size_t)toks[i0] * us_ld);
        const uint4* x1r = reinterpret_cast<const uint4*>(u_s + (size_t)toks[i1] * us_ld);
        float g0a = 0.f, g0b = 0.f, v0a = 0.f, v0b = 0.f, g1a = 0.f, g1b = 0.f, v1a = 0.f,
              v1b = 0.f;
        for (int c = b0 * 4; c < b1 * 4; ++c) {  // 8 elements per step
          // elements 8c .. 8c+7: block c / 4, offset o = 8 (c % 4) in the
          // block; byte j of a block holds element j (low nibble) and j + 16
          // (high nibble)
          const int blk = c >> 2, o = (c & 3) * 8;
          const int byte0 = blk * 16 + (o & 15);
          const uint2 gwd = *reinterpret_cast<const uint2*>(gq_r + byte0);
          const uint2 vwd = *reinterpret_cast<const uint2*>(vq_r + byte0);
          const float gsc = f16f(gs_r[blk]), vsc = f16f(vs_r[blk]);
          const int sh = o >= 16 ? 4 : 0;
          const uint32_t g_lo = (gwd.x >> sh) & 0x0F0F0F0Fu, g_hi = (gwd.y >> sh) & 0x0F0F0F0Fu;
          const uint32_t v_lo = (vwd.x >> sh) & 0x0F0F0F0Fu, v_hi = (vwd.y >> sh) & 0x0F0F0F0Fu;
          const uint4 xu = x0r[c], yu = x1r[c];
          float x[8], y[8];
          const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w}, yw[4] = {yu.x, yu.y, yu.z, yu.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 fx = __half22float2(*reinterpret_cast<const __half2*>(&xw[q]));
            const float2 fy = __half22float2(*reinterpret_cast<const __half2*>(&yw[q]));
            x[2 * q] = fx.x;
            x[2 * q + 1] = fx.y;
            y[2 * q] = fy.x;
            y[2 * q + 1] = fy.y;
          }
          float gv[8], vv[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // (q - 8) s, exact in fp32
            gv[q] = nib(g_lo, q) * gsc;
            gv[4 + q] = nib(g_hi, q) * gsc;
            vv[q] = nib(v_lo, q) * vsc;
            vv[4 + q] = nib(v_hi, q) * vsc;
          }
#pragma unroll
          for (int q = 0; q < 8; q += 2) {
            g0a = fmaf(gv[q], x[q], g0a);
            g0b = fmaf(gv[q + 1], x[q + 1], g0b);
            v0a = fmaf(vv[q], x[q], v0a);
            v0b = fmaf(vv[q + 1], x[q + 1], v0b);
            g1a = fmaf(gv[q], y[q], g1a);
            g1b = fmaf(gv[q + 1], y[q + 1], g1b);
            v1a = fmaf(vv[q], y[q], v1a);
            v1b = fmaf(vv[q + 1], y[q + 1], v1b);
          }
        }
        float* pr = part + ((size_t)(r * ne + i0) * nparts + pp) * 2;
        pr[0] = g0a + g0b;
        pr[1] = v0a + v0b;
        if (i1 != i0) {
          float* pq = part + ((size_t)(r * ne + i1) * nparts + pp) * 2;
          pq[0] = g1a + g1b;
          pq[1] = v1a + v1b;
        }
      }
      __syncthreads();
      if (it == b) stamp(p, l, 6);
      for (int v = tid; v < RA * ne; v += blockDim.x) {
        const int i = v / RA, r = v - i * RA;
        const float* pr = part + (size_t)(r * ne + i) * nparts * 2;
        float g = 0.f, vu = 0.f;
#pragma unroll 4
        for (int pp = 0; pp < nparts; ++pp) {
          g += pr[2 * pp];
          vu += pr[2 * pp + 1];
        }
        p.H[((size_t)e * T + toks[i]) * h + (size_t)sl * RA + r] = silu(g) * vu;
      }
    }
    if (b >= nitems)
      for (int i = 4; i < 7; ++i) stamp(p, l, i);
    stamp(p, l, 7);
    grid_arrive(p.bar);
    if (P.nbuf == 2 && !last)  // next layer's router rows, while the barrier completes
      stage_rows(sm + ((l & 1) ? P.wr0 : P.wr1), ws_ld * 4,
                 reinterpret_cast<const char*>(p.layer[l + 1].w_route), (size_t)d * 4, N, d * 4);
    cp_commit();  // the router rows' own group: phase B does not wait for it
    // aq / as are free until the next layer's phase A: stage block b's likely
    // item of the next layer now (its own group, waited for at the next
    // layer's start, not by phase B)
    spec = !last && Tk >= N && b < N * slicesA;
    if (spec) stage_rows_of(p.layer[l + 1], b / slicesA, b % slicesA);
    cp_commit();
    if (!grid_wait(p.bar, (unsigned)G * ++n_bar, p.status)) {
      cp_wait_all();
      return;
    }
    stamp(p, l, 8);

    // ---- phase B: y = sum_s a_s W_down[e_s] H_s, u_next = fp16(u + y), one
    // (token, RB output rows) unit at a time
    for (int un = b; un < nunits; un += G) {
      const int t = un / nsl, sl = un - t * nsl;
      if (un != b) {
        stage_unit(un);
        cp_commit();
        cp_wait_group<0>();
      } else {
        cp_wait_group<2>();  // this unit's rows; the next router rows and item may be in flight
      }
      __syncthreads();
      if (un == b) stamp(p, l, 9);
      // thread = (slot s, row group g, q4 block pp), pp fastest so a slot's
      // nbh partial dots sit in adjacent lanes; the RB rows are split into
      // rgroups groups so that about a CTA's worth of threads work
      int rgroups = 1;
      while (rgroups < RB && k * nbh * rgroups * 2 <= (int)blockDim.x) rgroups *= 2;
      const int rper = RB / rgroups;
      const int nthr = k * nbh * rgroups;
      for (int base = 0; base < nthr; base += blockDim.x) {  // uniform per warp
        const int uu = base + tid;
        const bool valid = uu < nthr;
        const int pp = uu % nbh, rest = uu / nbh;
        const int g = rest % rgroups, s2 = valid ? rest / rgroups : 0;
        const int e = sel[t * k + s2];
        float hc[32];
        if (valid) {
          const float4* hp =
              reinterpret_cast<const float4*>(p.H + ((size_t)e * T + t) * h + pp * 32);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 v = __ldcg(hp + c);
            hc[4 * c] = v.x;
            hc[4 * c + 1] = v.y;
            hc[4 * c + 2] = v.z;
            hc[4 * c + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) hc[c] = 0.f;
        }
        for (int r = g * rper; r < (g + 1) * rper; ++r) {
          // the block's sum of (q - 8) h times its scale
          float zz = 0.0f;
          if (valid)
            zz = f16f(bs[((size_t)s2 * RB + r) * nbh + pp]) *
                 q4_block_dot(bq + ((size_t)s2 * RB + r) * (h / 2) + pp * 16, hc);
          for (int o = nbh / 2; o >= 1; o >>= 1) zz += __shfl_xor_sync(0xffffffffu, zz, o);
          if (valid && pp == 0) zs[s2 * (RB + 1) + r] = zz;
        }
      }
      __syncthreads();
      if (un == b) stamp(p, l, 10);
      const bool early_next = P.early && !last;
      for (int r = tid; r < RB; r += blockDim.x) {
        float acc = 0.0f;
        for (int q = 0; q < k; ++q) acc = fmaf(aw[t * k + q], zs[q * (RB + 1) + r], acc);
        const int m = sl * RB + r;
        const size_t o = (size_t)t * d + m;
        if (last && p.y) p.y[o] = __float2half_rn(acc);
        const __half un = __float2half_rn(__half2float(u_s[(size_t)t * us_ld + m]) + acc);
        if (u_next) u_next[o] = un;
        if (early_next) part[r] = __half2float(un);
      }
      if (early_next) {
        // the next layer's router block sums of this unit's kRouteBlock-wide
        // blocks of u_{l+1}[t]: one ascending FMA chain per (expert, block)
        // over the prefetched router rows, stored for every CTA to read
        cp_wait_group<1>();  // the next router rows (the speculative item may be in flight)
        __syncthreads();
        const float* wn = reinterpret_cast<const float*>(sm + ((l & 1) ? P.wr0 : P.wr1));
        for (int q = tid; q < N * (RB / kRouteBlock); q += blockDim.x) {
          const int i = q % N, mb = q / N;
          const int j0 = sl * RB + mb * kRouteBlock;
          const float4* w4 = reinterpret_cast<const float4*>(wn + (size_t)i * ws_ld + j0);
          const float4* x4 = reinterpret_cast<const float4*>(part + mb * kRouteBlock);
          float c = 0.0f;
#pragma unroll 8
          for (int s4 = 0; s4 < kRouteBlock / 4; ++s4) {
            const float4 w = w4[s4], x = x4[s4];
            c = __fmaf_rn(w.x, x.x, c);
            c = __fmaf_rn(w.y, x.y, c);
            c = __fmaf_rn(w.z, x.z, c);
            c = __fmaf_rn(w.w, x.w, c);
          }
          p.zb[((size_t)(j0 / kRouteBlock) * N + i) * T + t] = c;
        }
      }
      __syncthreads();
    }
    if (b >= nunits)
      for (int i = 9; i < 11; ++i) stamp(p, l, i);
    stamp(p, l, 11);
    grid_arrive(p.bar);
    if (!grid_wait(p.bar, (unsigned)G * ++n_bar, p.status)) {
      cp_wait_all();
      return;
    }
    stamp(p, l, 12);
  }
}

// ================================================ per-token decode kernel
// Tokens are independent through the layer stack, so this kernel needs no
// grid barrier.  CTA b owns the item (token t, slot s, hidden slice j of S)
// for every layer (T k S CTAs, at most one per SM) and keeps its token's
// row u_l[t] in shared memory.  Per layer it routes token t itself (the
// 128-input block chains of its logits, top-k), stages the selected
// expert's gate and up rows of slice j and the slice's down columns, forms
// H_j = SiLU(W_gate u) * (W_up u) on chip and the partial output row
// W_down[:, slice j] H_j in its own shared memory.  A token's k S CTAs form
// one thread-block cluster: after a cluster barrier each of them reads the
// token's k S partial rows from the cluster's shared memory and sums them in
// one fixed order (slots in order, each slot's slices in order) into
// u_{l+1}[t] = fp16(u_l + y), so all of them hold the same next row and
// route it to the same experts.  Partial rows alternate between two buffers
// by layer parity: a CTA passes the next layer's cluster barrier only after
// every peer has read this layer's rows.  Nothing waits across clusters, so
// the launch needs no co-residency beyond the cluster's.  Only the selected
// experts' rows are read.
struct Plan2 {
  int S;       // hidden slices per (token, slot)
  int hS;      // hidden units per slice
  int nparts;  // parts of d per gate/up row (one thread each)
  uint32_t wr, z, sel, aw, zp, uh, uf, gq, gs, dq, ds, part, hs, yr, misc;
  uint32_t total;
};

struct Params2 {
  LayerPtrs layer[kLayersPerLaunch];
  int n_layers;
  int T, d, N, k, h, renorm;
  Plan2 plan;
  const __half* u_in;
  __half* u_out;
  __half* y;
  int32_t* top_idx;
  float* top_w;
  unsigned long long* stamps;
};

// Stamps of the per-token kernel, in the same 13 slots (block 0's item):
// 0 layer start, 1 = 0, 2 routed, 3 = 2, 4 the item's gate/up rows staged,
// 5 = 4, 6 gate/up dots formed, 7 H formed, 8 = 7, 9 down columns ready,
// 10 partial row in shared memory, 11 cluster barrier passed (every row of
// the token there), 12 next row formed.
__device__ __forceinline__ void stamp2(const Params2& p, int l, int i) {
  if (p.stamps && blockIdx.x == 0 && threadIdx.x == 0)
    p.stamps[(size_t)l * kStamps + i] = clock64();
}

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned start and size).
__device__ __forceinline__ void l2_prefetch(const void* ptr, int bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

// Shared row stride of a down row's slice (hS / 2 bytes): padded by 16 bytes
// when it is a multiple of 32, so the 16-byte loads of a warp's 32 rows hit
// distinct banks.
__host__ __device__ __forceinline__ int dq_ld(int hS) {
  return (hS / 2) % 32 == 0 ? hS / 2 + 16 : hS / 2;
}

bool make_plan2(const moe_shape& s, int sms, Plan2* out) {
  const int T = s.T, d = s.d, N = s.N, k = s.k, h = s.h;
  const int nb = d / 32, nbh = h / 32, nblk = (d + kRouteBlock - 1) / kRouteBlock;
  if ((int64_t)T * k > sms || k > 8) return false;  // one CTA per item, clusters <= 8
  // the most slices that keep one CTA per item and k S within a portable
  // cluster
  int S0 = 1;
  while (2 * S0 <= nbh && (int64_t)T * k * 2 * S0 <= sms && k * 2 * S0 <= 8) S0 *= 2;
  for (int S = S0; S >= 1; S /= 2) {
    const int hS = h / S;
    if (2 * hS > kThreads) break;
    Plan2 p{};
    p.S = S;
    p.hS = hS;
    p.nparts = kThreads / (2 * hS);
    if (p.nparts > nb) p.nparts = nb;
    uint32_t off = 0;
    p.wr = take(off, (size_t)N * (d + 4) * 4);
    p.z = take(off, (size_t)N * 4);
    p.sel = take(off, (size_t)k * 4);
    p.aw = take(off, (size_t)k * 4);
    p.zp = take(off, (size_t)N * nblk * 4);
    p.uh = take(off, (size_t)d * 2);
    p.uf = take(off, (size_t)d * 4);
    p.gq = take(off, (size_t)2 * hS * (d / 2 + 16));  // rows padded 16 B: no bank conflicts
    p.gs = take(off, (size_t)2 * hS * nb * 2);
    p.dq = take(off, (size_t)d * dq_ld(hS));
    p.ds = take(off, (size_t)d * nbh * 2);
    p.part = take(off, (size_t)2 * hS * p.nparts * 4);
    p.hs = take(off, (size_t)hS * 4);
    p.yr = take(off, (size_t)2 * d * 4);
    p.misc = take(off, 16);
    p.total = off;
    if (off <= kSmemLimit) {
      *out = p;
      return true;
    }
  }
  return false;
}

// Cluster barrier of all threads (release / acquire, so shared-memory stores
// before it are seen by the cluster's loads after it), a shared-memory
// address of the cluster's CTA `rank`, and a load from it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads, 1) decode_token(const __grid_constant__ Params2 p) {
  extern __shared__ __align__(16) char sm[];
  const Plan2& P = p.plan;
  const int T = p.T, d = p.d, N = p.N, k = p.k, h = p.h, Tk = T * k;
  const int S = P.S, hS = P.hS, nparts = P.nparts, KS = k * S;
  const int nb = d / 32, nbh = h / 32, nblk = (d + kRouteBlock - 1) / kRouteBlock;
  const int ws_ld = d + 4, cpr = hS / 32;
  const int b = blockIdx.x, tid = threadIdx.x;
  float* wr = reinterpret_cast<float*>(sm + P.wr);
  float* z = reinterpret_cast<float*>(sm + P.z);
  int* sel = reinterpret_cast<int*>(sm + P.sel);
  float* aw = reinterpret_cast<float*>(sm + P.aw);
  float* zp = reinterpret_cast<float*>(sm + P.zp);
  __half* uh = reinterpret_cast<__half*>(sm + P.uh);
  float* uf = reinterpret_cast<float*>(sm + P.uf);
  uint8_t* gq = reinterpret_cast<uint8_t*>(sm + P.gq);
  uint16_t* gs = reinterpret_cast<uint16_t*>(sm + P.gs);
  uint8_t* dq = reinterpret_cast<uint8_t*>(sm + P.dq);
  uint16_t* ds = reinterpret_cast<uint16_t*>(sm + P.ds);
  float* part = reinterpret_cast<float*>(sm + P.part);
  float* hsv = reinterpret_cast<float*>(sm + P.hs);
  float* yr = reinterpret_cast<float*>(sm + P.yr);
  if (b >= Tk * S) return;  // (the grid is exactly T k S)
  const int pr = b / S, j = b - pr * S, t = pr / k, s = pr - t * k;
  const bool writer = s == 0 && j == 0;  // writes the token's routing and outputs

  // the token's input row and layer 0's router rows
  stage_bytes(uh, p.u_in + (size_t)t * d, d * 2);
  stage_rows(reinterpret_cast<char*>(wr), ws_ld * 4,
             reinterpret_cast<const char*>(p.layer[0].w_route), (size_t)d * 4, N, d * 4);
  cp_wait_all();
  __syncthreads();
  for (int i = tid; i < d; i += blockDim.x) uf[i] = __half2float(uh[i]);
  __syncthreads();
  for (int l = 0; l < p.n_layers; ++l) {
    const LayerPtrs& L = p.layer[l];
    const bool last = l == p.n_layers - 1;
    stamp2(p, l, 0);
    stamp2(p, l, 1);
    // ---- route token t: block chains over its row, sums in block order, top-k
    for (int q = tid; q < N * nblk; q += blockDim.x) {
      const int i = q % N, m = q / N, j0 = m * kRouteBlock;
      const int len = min(kRouteBlock, d - j0);
      const float4* w4 = reinterpret_cast<const float4*>(wr + (size_t)i * ws_ld + j0);
      const float4* x4 = reinterpret_cast<const float4*>(uf + j0);
      float c = 0.0f;
#pragma unroll 4
      for (int s4 = 0; s4 < len / 4; ++s4) {
        const float4 wv = w4[s4], x = x4[s4];
        c = __fmaf_rn(wv.x, x.x, c);
        c = __fmaf_rn(wv.y, x.y, c);
        c = __fmaf_rn(wv.z, x.z, c);
        c = __fmaf_rn(wv.w, x.w, c);
      }
      zp[m * N + i] = c;
    }
    __syncthreads();
    for (int i = tid; i < N; i += blockDim.x) {
      float zz = 0.0f;
      for (int m = 0; m < nblk; ++m) zz = __fadd_rn(zz, zp[m * N + i]);
      z[i] = L.bias ? __fadd_rn(zz, L.bias[i]) : zz;
    }
    __syncthreads();
    if (tid == 0) {
      if (N == 8 && k == 2)
        topk8_k2(z, p.renorm, sel, aw);
      else if (N <= 8)
        topk_token<8>(z, N, k, p.renorm, sel, aw);
      else if (N <= 32)
        topk_token<32>(z, N, k, p.renorm, sel, aw);
      else
        topk_wide(z, N, k, p.renorm, sel, aw);
    }
    __syncthreads();
    if (writer)
      for (int x = tid; x < k; x += blockDim.x) {
        if (p.top_idx) p.top_idx[(size_t)l * Tk + t * k + x] = sel[x];
        if (last && p.top_w) p.top_w[t * k + x] = aw[x];
      }
    stamp2(p, l, 2);
    stamp2(p, l, 3);
    const int e = sel[s];
    // ---- the slice's gate and up rows (one group), its down columns
    // (another), the next layer's router rows (a third; routing above was
    // the last reader of the buffer)
    const size_t grow = (size_t)e * h + (size_t)j * hS;
    stage_rows(reinterpret_cast<char*>(gq), d / 2 + 16,
               reinterpret_cast<const char*>(L.gq + grow * (d / 2)), d / 2, hS, d / 2);
    stage_rows(reinterpret_cast<char*>(gq) + (size_t)hS * (d / 2 + 16), d / 2 + 16,
               reinterpret_cast<const char*>(L.uq + grow * (d / 2)), d / 2, hS, d / 2);
    stage_bytes(gs, L.gs + grow * nb, hS * nb * 2);
    stage_bytes(gs + (size_t)hS * nb, L.us + grow * nb, hS * nb * 2);
    cp_commit();
    stage_rows(reinterpret_cast<char*>(dq), dq_ld(hS),
               reinterpret_cast<const char*>(L.dq + (size_t)e * d * (h / 2) + (size_t)j * (hS / 2)),
               h / 2, d, hS / 2);
    stage_bytes(ds, L.ds + (size_t)e * d * nbh, d * nbh * 2);
    cp_commit();
    if (!last)
      stage_rows(reinterpret_cast<char*>(wr), ws_ld * 4,
                 reinterpret_cast<const char*>(p.layer[l + 1].w_route), (size_t)d * 4, N,
                 d * 4);
    cp_commit();
    cp_wait_group<2>();  // the gate/up rows
    __syncthreads();
    stamp2(p, l, 4);
    stamp2(p, l, 5);
    // ---- gate/up dots: thread = (row r2 of the 2 hS gate/up rows, part pp
    // of d); per q4 block the sum of (q - 8) x, then one multiply-add by the
    // block scale
    for (int u2 = tid; u2 < 2 * hS * nparts; u2 += blockDim.x) {
      const int r2 = u2 % (2 * hS), pp = u2 / (2 * hS);
      const int b0 = pp * nb / nparts, b1 = (pp + 1) * nb / nparts;
      const uint8_t* q = gq + (size_t)r2 * (d / 2 + 16);
      const uint16_t* sc = gs + (size_t)r2 * nb;
      float acc = 0.0f;
#pragma unroll 2
      for (int blk = b0; blk < b1; ++blk) {
        const uint4 raw = *reinterpret_cast<const uint4*>(q + blk * 16);
        const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
        const float4* x4 = reinterpret_cast<const float4*>(uf + blk * 32);
        float c0 = 0.0f, c1 = 0.0f, c2 = 0.0f, c3 = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t lo = wd[i] & 0x0F0F0F0Fu, hi = (wd[i] >> 4) & 0x0F0F0F0Fu;
          const float4 xl = x4[i], xh = x4[4 + i];  // elements 4i.. and 16+4i..
          c0 = fmaf(nib(lo, 0), xl.x, c0);
          c1 = fmaf(nib(lo, 1), xl.y, c1);
          c2 = fmaf(nib(lo, 2), xl.z, c2);
          c3 = fmaf(nib(lo, 3), xl.w, c3);
          c0 = fmaf(nib(hi, 0), xh.x, c0);
          c1 = fmaf(nib(hi, 1), xh.y, c1);
          c2 = fmaf(nib(hi, 2), xh.z, c2);
          c3 = fmaf(nib(hi, 3), xh.w, c3);
        }
        acc = fmaf(f16f(sc[blk]), (c0 + c1) + (c2 + c3), acc);
      }
      part[r2 * nparts + pp] = acc;
    }
    __syncthreads();
    stamp2(p, l, 6);
    for (int r = tid; r < hS; r += blockDim.x) {
      float g = 0.0f, v = 0.0f;
      for (int pp = 0; pp < nparts; ++pp) {
        g += part[r * nparts + pp];
        v += part[(hS + r) * nparts + pp];
      }
      hsv[r] = silu(g) * v;
    }
    cp_wait_group<1>();  // the down columns
    __syncthreads();
    stamp2(p, l, 7);
    stamp2(p, l, 8);
    stamp2(p, l, 9);
    // ---- partial output row: row o of W_down[e] over the slice's hidden
    // units, into this CTA's buffer of the layer's parity
    // A thread takes rows o0 and o0 + blockDim.x together, so each H value
    // it loads feeds both; per q4 block the sum of (q - 8) h, then one
    // multiply-add by the block scale.
    float* ymine = yr + (size_t)(l & 1) * d;
    const int dld = dq_ld(hS);
    for (int o0 = tid; o0 < d; o0 += 2 * blockDim.x) {
      const int o1 = o0 + blockDim.x < d ? o0 + blockDim.x : o0;
      const uint8_t* q0 = dq + (size_t)o0 * dld;
      const uint8_t* q1 = dq + (size_t)o1 * dld;
      const uint16_t* s0 = ds + (size_t)o0 * nbh + (size_t)j * cpr;
      const uint16_t* s1 = ds + (size_t)o1 * nbh + (size_t)j * cpr;
      float y0 = 0.0f, y1 = 0.0f;
#pragma unroll 2
      for (int bl = 0; bl < cpr; ++bl) {
        const uint4 r0 = *reinterpret_cast<const uint4*>(q0 + bl * 16);
        const uint4 r1 = *reinterpret_cast<const uint4*>(q1 + bl * 16);
        const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
        const float4* h4 = reinterpret_cast<const float4*>(hsv + bl * 32);
        float c00 = 0.0f, c01 = 0.0f, c10 = 0.0f, c11 = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t lo0 = w0[i] & 0x0F0F0F0Fu, hi0 = (w0[i] >> 4) & 0x0F0F0F0Fu;
          const uint32_t lo1 = w1[i] & 0x0F0F0F0Fu, hi1 = (w1[i] >> 4) & 0x0F0F0F0Fu;
          const float4 hl = h4[i], hh = h4[4 + i];  // elements 4i.. and 16+4i..
          c00 = fmaf(nib(lo0, 0), hl.x, c00);
          c10 = fmaf(nib(lo1, 0), hl.x, c10);
          c01 = fmaf(nib(lo0, 1), hl.y, c01);
          c11 = fmaf(nib(lo1, 1), hl.y, c11);
          c00 = fmaf(nib(lo0, 2), hl.z, c00);
          c10 = fmaf(nib(lo1, 2), hl.z, c10);
          c01 = fmaf(nib(lo0, 3), hl.w, c01);
          c11 = fmaf(nib(lo1, 3), hl.w, c11);
          c00 = fmaf(nib(hi0, 0), hh.x, c00);
          c10 = fmaf(nib(hi1, 0), hh.x, c10);
          c01 = fmaf(nib(hi0, 1), hh.y, c01);
          c11 = fmaf(nib(hi1, 1), hh.y, c11);
          c00 = fmaf(nib(hi0, 2), hh.z, c00);
          c10 = fmaf(nib(hi1, 2), hh.z, c10);
          c01 = fmaf(nib(hi0, 3), hh.w, c01);
          c11 = fmaf(nib(hi1, 3), hh.w, c11);
        }
        y0 = fmaf(f16f(s0[bl]), c00 + c01, y0);
        y1 = fmaf(f16f(s1[bl]), c10 + c11, y1);
      }
      ymine[o0] = y0;
      if (o1 != o0) ymine[o1] = y1;
    }
    stamp2(p, l, 10);
    // while the cluster meets: CTA b < N S pulls the next layer's gate/up
    // rows of (expert b / S, slice b % S) into L2
    if (!last && b < N * S && tid == 0) {
      const LayerPtrs& Ln = p.layer[l + 1];
      const int ep = b / S, jp = b - (b / S) * S;
      const size_t gp = (size_t)ep * h + (size_t)jp * hS;
      l2_prefetch(Ln.gq + gp * (d / 2), hS * (d / 2));
      l2_prefetch(Ln.uq + gp * (d / 2), hS * (d / 2));
      if (jp == 0) l2_prefetch(Ln.dq + (size_t)ep * d * (h / 2), d * (h / 2));
    }
    cluster_sync_all();  // every partial row of the token is in the cluster
    stamp2(p, l, 11);
    // ---- the token's next row, the same in each of its CTAs: cluster rank
    // s2 S + j2 holds slot s2's slice j2
    const uint32_t ymine_a = static_cast<uint32_t>(__cvta_generic_to_shared(ymine));
    const int lgS = __ffs(S) - 1;
    for (int o = tid; o < d; o += blockDim.x) {
      // the k S rows' values of column o, loaded together, then summed in order
      float yv[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        yv[r] = r < KS ? ld_cluster_f32(cluster_addr(ymine_a + 4u * o, r)) : 0.0f;
      float acc = 0.0f, ys = 0.0f;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < KS) {
          ys += yv[r];
          if (((r + 1) & (S - 1)) == 0) {  // slot r / S complete (S a power of 2)
            acc = fmaf(aw[r >> lgS], ys, acc);
            ys = 0.0f;
          }
        }
      }
      const __half un = __float2half_rn(__half2float(uh[o]) + acc);
      if (last && writer) {
        if (p.y) p.y[(size_t)t * d + o] = __float2half_rn(acc);
        if (p.u_out) p.u_out[(size_t)t * d + o] = un;
      }
      uh[o] = un;
      uf[o] = __half2float(un);
    }
    cp_wait_group<0>();  // the next layer's router rows
    __syncthreads();
    stamp2(p, l, 12);
  }
  cluster_sync_all();  // no CTA leaves while a peer may still read its rows
}

// ------------------------------------------------------------------ host
struct WsLayout {
  float* H;
  float* zb;
  int32_t* idx;
  float* w;
  __half* work;
  unsigned* bar;  // [0] arrivals, [1] abort of the two-phase kernel's barriers
  size_t bytes;
};

WsLayout carve_decode(const moe_shape& s, void* base) {
  Carver c(base);
  WsLayout L;
  L.H = c.take<float>((size_t)s.N * s.T * s.h);
  L.zb = c.take<float>((size_t)((s.d + kRouteBlock - 1) / kRouteBlock) * s.N * s.T);
  L.idx = c.take<int32_t>((size_t)s.T * s.k);
  L.w = c.take<float>((size_t)s.T * s.k);
  L.work = c.take<__half>((size_t)s.T * s.d);
  L.bar = c.take<unsigned>(4);
  L.bytes = c.used();
  return L;
}

// SM count of the current device; the kernel's shared-memory limit is raised
// once per device.
bool device_info(int* sms) {
  static std::atomic<int> sm_count[kMaxDevices];
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || !device_slot(dev)) return false;
  if (needs_setup(configured, dev)) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaFuncSetAttribute(decode_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemLimit) != cudaSuccess ||
        cudaFuncSetAttribute(decode_token, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemLimit) != cudaSuccess)
      return false;
    MOE_PREFER_SHARED((decode_persistent));
    MOE_PREFER_SHARED((decode_token));
    sm_count[dev].store(n, std::memory_order_relaxed);
    mark_setup(configured, dev);
  }
  *sms = sm_count[dev].load(std::memory_order_relaxed);
  return true;
}

bool decode_shape_ok(const moe_shape* s) {
  if (!shape_ok(s) || s->T > kMaxT || s->N > kMaxN || s->k > 8 || s->d % 32 != 0 ||
      s->h % 32 != 0 || (s->h / 32) > 32 || 32 % (s->h / 32) != 0)
    return false;
  // Plan with the current device's SM count, as launch_decode does (fewer
  // SMs take more rows per CTA and more shared memory); 148 (B200) when no
  // device is visible, where nothing can be launched anyway.
  int sms = 0;
  if (!device_info(&sms) || sms <= 0) sms = 148;
  Plan p;
  return make_plan(*s, sms, &p);
}

bool aligned4(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 3u) == 0; }

bool layer_ok(const moe_q4_layer* L) {
  return L && L->w_route && L->gate_qs && L->gate_scales && L->up_qs && L->up_scales &&
         L->down_qs && L->down_scales && aligned16(L->gate_qs) && aligned16(L->up_qs) &&
         aligned16(L->down_qs) && aligned16(L->w_route) && aligned4(L->gate_scales) &&
         aligned4(L->up_scales) && aligned4(L->down_scales) && aligned4(L->bias);
}

LayerPtrs layer_ptrs(const moe_q4_layer& L) {
  return LayerPtrs{L.w_route, L.bias, L.gate_qs, L.gate_scales,
                   L.up_qs,   L.up_scales, L.down_qs, L.down_scales};
}

enum class DecodeKind { kNone = 0, kPerToken = 1, kTwoPhase = 2 };

// Launch configuration of the per-token kernel: T k S CTAs in clusters of
// k S (one token each); attr must outlive the returned configuration.
cudaLaunchConfig_t token_launch_cfg(const moe_shape& s, const Plan2& plan, cudaStream_t st,
                                    cudaLaunchAttribute* attr) {
  const int ks = s.k * plan.S;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.T * ks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan.total;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// The per-token kernel over layers [0, n): T k S CTAs, one item each, in
// clusters of k S (one token each).
int launch_decode_token(const moe_shape& s, const Plan2& plan, const moe_q4_layer* layers, int n,
                        const __half* u_in, __half* u_out, __half* y, int32_t* top_idx,
                        float* top_w, cudaStream_t st, unsigned long long* stamps) {
  Params2 p{};
  p.plan = plan;
  for (int l = 0; l < n; ++l) p.layer[l] = layer_ptrs(layers[l]);
  p.n_layers = n;
  p.T = s.T;
  p.d = s.d;
  p.N = s.N;
  p.k = s.k;
  p.h = s.h;
  p.renorm = s.renorm;
  p.u_in = u_in;
  p.u_out = u_out;
  p.y = y;
  p.top_idx = top_idx;
  p.top_w = top_w;
  p.stamps = stamps;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = token_launch_cfg(s, plan, st, attr);
  return cudaLaunchKernelEx(&cfg, decode_token, p) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Which kernel a shape runs on this device: the per-token kernel when its
// plan fits and a cluster of the token's k S CTAs can be resident, else the
// two-phase kernel when its plan fits, else none.
DecodeKind choose_decode(const moe_shape& s, int sms, Plan2* plan2) {
  if (make_plan2(s, sms, plan2)) {
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = token_launch_cfg(s, *plan2, nullptr, attr);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, decode_token, &cfg) == cudaSuccess &&
        clusters >= 1)
      return DecodeKind::kPerToken;
    cudaGetLastError();  // clear the error a failed query recorded
  }
  Plan p;
  return make_plan(s, sms, &p) ? DecodeKind::kTwoPhase : DecodeKind::kNone;
}

// One launch over layers [0, n) of `layers`: the per-token kernel (thread-
// block clusters, one per token) when its items fit one per SM and its
// shared-memory plan fits, else the cooperative two-phase kernel.
int launch_decode(const moe_shape& s, const moe_q4_layer* layers, int n, const __half* u_in,
                  __half* u_out, __half* y, int32_t* top_idx, float* top_w, const WsLayout& W,
                  cudaStream_t st, unsigned long long* stamps = nullptr) {
  int sms = 0;
  if (!device_info(&sms)) return MOE_ERR_CUDA;
  Plan2 plan2;
  const DecodeKind kind = choose_decode(s, sms, &plan2);
  if (kind == DecodeKind::kNone) return MOE_ERR_UNSUPPORTED;
  if (kind == DecodeKind::kPerToken)
    return launch_decode_token(s, plan2, layers, n, u_in, u_out, y, top_idx, top_w, st, stamps);
  Params p{};
  if (!make_plan(s, sms, &p.plan)) return MOE_ERR_UNSUPPORTED;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_persistent, kThreads,
                                                    p.plan.total) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (occ < 1) return MOE_ERR_UNSUPPORTED;
  const int items = p.plan.nsel_max * (s.h / p.plan.RA), slices = s.T * (s.d / p.plan.RB);
  int grid = items > slices ? items : slices;
  if (grid > sms) grid = sms;
  for (int l = 0; l < n; ++l) p.layer[l] = layer_ptrs(layers[l]);
  p.n_layers = n;
  p.T = s.T;
  p.d = s.d;
  p.N = s.N;
  p.k = s.k;
  p.h = s.h;
  p.renorm = s.renorm;
  p.u_in = u_in;
  p.u_work = W.work;
  p.u_out = u_out;
  p.y = y;
  p.top_idx = top_idx;
  p.top_w = top_w;
  p.H = W.H;
  p.zb = W.zb;
  p.bar = W.bar;
  p.status = status_word();
  p.stamps = stamps;
  if (cudaMemsetAsync(W.bar, 0, 4 * sizeof(unsigned), st) != cudaSuccess) return MOE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.plan.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_persistent, p) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace
}  // namespace moe

extern "C" int moe_decode_kernel(const moe_shape* shape) {
  if (!moe::decode_shape_ok(shape)) return 0;
  int sms = 0;
  if (!moe::device_info(&sms) || sms <= 0) return 0;
  moe::Plan2 plan2;
  return static_cast<int>(moe::choose_decode(*shape, sms, &plan2));
}

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
  if (shape->T == 0) return MOE_OK;
  return launch_decode(*shape, layer, 1, reinterpret_cast<const __half*>(u),
                       reinterpret_cast<__half*>(u_next), reinterpret_cast<__half*>(y),
                       top_idx ? top_idx : W.idx, top_w ? top_w : W.w, W, as_stream(stream));
}

namespace {
int decode_step(const moe_shape* shape, int32_t n_layers, const moe_q4_layer* layers,
                const uint16_t* u0, uint16_t* u_out, int32_t* top_idx_all, void* ws,
                size_t ws_bytes, void* stream, uint64_t* stamps) {
  using namespace moe;
  if (!decode_shape_ok(shape) || n_layers <= 0 || !layers) return MOE_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    if (!layer_ok(&layers[l])) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!u0 || !u_out)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u0) || !aligned16(u_out)) return MOE_ERR_INVALID_ARG;
  WsLayout W = carve_decode(*shape, ws);
  if (!ws || ws_bytes < W.bytes) return MOE_ERR_WORKSPACE;
  if (shape->T == 0) return MOE_OK;
  const moe_shape& s = *shape;
  cudaStream_t st = as_stream(stream);
  const size_t Tk = (size_t)s.T * s.k;
  for (int l0 = 0; l0 < n_layers; l0 += kLayersPerLaunch) {
    const int n = n_layers - l0 < kLayersPerLaunch ? n_layers - l0 : kLayersPerLaunch;
    const bool last_chunk = l0 + n == n_layers;
    const __half* in = l0 == 0 ? reinterpret_cast<const __half*>(u0) : W.work;
    __half* out = last_chunk ? reinterpret_cast<__half*>(u_out) : W.work;
    const int rc = launch_decode(
        s, layers + l0, n, in, out, nullptr, top_idx_all ? top_idx_all + l0 * Tk : nullptr,
        nullptr, W, st,
        stamps ? reinterpret_cast<unsigned long long*>(stamps) + (size_t)l0 * kStamps : nullptr);
    if (rc != MOE_OK) return rc;
  }
  return MOE_OK;
}
}  // namespace

extern "C" int moe_decode_step(const moe_shape* shape, int32_t n_layers,
                               const moe_q4_layer* layers, const uint16_t* u0, uint16_t* u_out,
                               int32_t* top_idx_all, void* ws, size_t ws_bytes, void* stream) {
  return decode_step(shape, n_layers, layers, u0, u_out, top_idx_all, ws, ws_bytes, stream,
                     nullptr);
}

extern "C" int moe_decode_step_trace(const moe_shape* shape, int32_t n_layers,
                                     const moe_q4_layer* layers, const uint16_t* u0,
                                     uint16_t* u_out, int32_t* top_idx_all, void* ws,
                                     size_t ws_bytes, uint64_t* stamps, void* stream) {
  if (!stamps || (reinterpret_cast<uintptr_t>(stamps) & 7u)) return MOE_ERR_INVALID_ARG;
  return decode_step(shape, n_layers, layers, u0, u_out, top_idx_all, ws, ws_bytes, stream,
                     stamps);
}
