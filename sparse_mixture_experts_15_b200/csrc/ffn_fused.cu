// Fused grouped SwiGLU expert FFN for small hidden widths on tcgen05.
//
// Tutorial "Mixture of Experts MoE: how sparse activation saves compute",
// §3.1 equation F: y = W_down (SiLU(W_gate x) * W_up x), per expert on its own
// grouped rows (§3.6).  When the hidden width h is small (h <= 256) one CTA
// can hold a token tile's whole hidden vector, so both GEMMs run in one
// launch and H never goes to HBM:
//
//   phase A  for each 64-wide hidden slice m: TMEM acc_A[m] = [64 gate rows;
//            64 up rows of slice m] x X_tile^T (K = width), TMA-staged
//   epilogue A  H = act(g, u) -> bf16, written by the epilogue warps straight
//            into shared memory in the 128-byte-swizzled K-major layout the
//            tensor core reads (then a generic->async proxy fence)
//   phase B  for each 128-wide output slice: TMEM acc_B = W_down rows x
//            H_tile^T (K = h), A by TMA, B from that shared-memory tile
//   epilogue B  y_rows fp32
//
// Same orientation as the two-launch kernel (weights on the MMA's M side,
// up to 64 tokens of one expert on N), persistent CTAs, one TMA producer
// thread, one MMA thread, four epilogue warps, bounded mbarrier waits.
#include <cuda.h>

#include "common.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace {

constexpr int fBM = 128, fBK = 64, fBN = 64, fS = 7, fThreads = 192, fEpiLd = 33;
constexpr int fHMax = 256;
// mbarriers after the stage ring: a_done per hidden slice (h / 64 <= 4),
// h_ready, b_done per output slice (width / 128 <= 8), b_free, drain
constexpr int kMaxA = fHMax / 64, kMaxB = 8, kBars = kMaxA + 1 + kMaxB + 2;
constexpr long long fWaitBudget = 4000000000LL;

struct FusedParams {
  CUtensorMap map_g;  // W_gate [G*h][width], box 64 x 64
  CUtensorMap map_u;  // W_up   [G*h][width], box 64 x 64
  CUtensorMap map_x;  // x_rows [R][width],   box 64 x fBN
  CUtensorMap map_d;  // W_down [G*width][h], box 64 x 128
  const int32_t* offsets;
  int R;  // rows of x_rows and y_rows
  int G, width, h;
  float beta_g, beta_u;
  void* y_rows;         // [R][width] fp32 (weighted by row_w when it is set)
  const float* row_w;   // nullable: combine weight of each grouped row
  int* status;
};

struct FLayout {
  static constexpr int A_BYTES = fBM * fBK * 2;  // 16 KB
  static constexpr int X_BYTES = fBN * fBK * 2;  // 8 KB
  static constexpr int STAGE = A_BYTES + X_BYTES;
  static constexpr int H_BYTES = fBN * fHMax * 2;  // 32 KB
  static constexpr int EPI_BYTES = fBM * fEpiLd * 4 + fBN * 4;  // exchange tile + row weights
  static size_t bytes(int G) {
    size_t b = 1024 + (size_t)fS * STAGE + H_BYTES + EPI_BYTES + (size_t)3 * (G + 1) * 4;
    b = align_up(b, 8);
    b += (size_t)(2 * fS + kBars) * 8 + 16;
    return b;
  }
};

__device__ __forceinline__ bool all_epi_ok(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

template <int ACT>
__global__ void __launch_bounds__(fThreads, 1) tc_fused_ffn(const __grid_constant__ FusedParams p) {
  using L = FLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  uint8_t* hs = smem + fS * L::STAGE;  // H tile, 1024-aligned (fS * STAGE is)
  float* epi = reinterpret_cast<float*>(hs + L::H_BYTES);
  float* fac = epi + fBM * fEpiLd;  // [fBN] the tile's combine weights
  int* grp_beg = reinterpret_cast<int*>(fac + fBN);
  int* grp_cnt = grp_beg + (p.G + 1);
  int* grp_pre = grp_cnt + (p.G + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(grp_pre + p.G + 1) + 7) & ~static_cast<uintptr_t>(7));
  uint64_t* full = bars;
  uint64_t* empty = bars + fS;
  uint64_t* a_done = bars + 2 * fS;  // [kMaxA]: slice m's gate/up accumulators ready
  uint64_t* h_ready = a_done + kMaxA;
  uint64_t* b_done = h_ready + 1;    // [kMaxB]: output slice m2's accumulator ready
  uint64_t* b_free = b_done + kMaxB;
  uint64_t* drain = b_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * fS + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int s = 0; s < fS; ++s) {
      tc::mbar_init(tc::smem_u32(&full[s]), 1);
      tc::mbar_init(tc::smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < kMaxA; ++i) tc::mbar_init(tc::smem_u32(&a_done[i]), 1);
    tc::mbar_init(tc::smem_u32(h_ready), 128);
    for (int i = 0; i < kMaxB; ++i) tc::mbar_init(tc::smem_u32(&b_done[i]), 1);
    tc::mbar_init(tc::smem_u32(b_free), 128);
    tc::mbar_init(tc::smem_u32(drain), 1);
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&p.map_g);
    tc::tma_prefetch_desc(&p.map_u);
    tc::tma_prefetch_desc(&p.map_x);
    tc::tma_prefetch_desc(&p.map_d);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::tmem_relinquish();
  }
  pdl_wait();
  pdl_allow_next();
  if (warp == 0) {  // group table: one tile = (expert, 64 tokens), all of h and width
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int g = base + lane;
      int beg = 0, cnt = 0;
      if (g < p.G) {
        beg = p.offsets[g];
        cnt = p.offsets[g + 1] - beg;
        if (cnt < 0 || beg < 0 || beg > p.R || cnt > p.R - beg) {  // rows outside the buffers
          record_error(p.status, MOE_ERR_BOUNDS);
          cnt = 0;
        }
      }
      const int t = g < p.G ? (cnt + fBN - 1) / fBN : 0;
      int incl = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (g < p.G) {
        grp_beg[g] = beg;
        grp_cnt[g] = cnt;
        grp_pre[g] = carry + incl - t;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) grp_pre[p.G] = carry;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = grp_pre[p.G];
  const int mA = p.h / 64, mB = p.width / fBM, kA = p.width / fBK, kB = p.h / fBK;

  auto decode = [&](int tile, int& g, int& n) {
    int lo = 0, hi = p.G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (grp_pre[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
    n = tile - grp_pre[g];
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int g, n;
        decode(tile, g, n);
        const int tok0 = grp_beg[g] + n * fBN;
        for (int j = 0; j < mA * kA + mB * kB && ok; ++j) {
          if (!tc::mbar_wait(tc::smem_u32(&empty[stage]), phase ^ 1u, abort_flag, fWaitBudget)) {
            ok = false;
            break;
          }
          const uint32_t fb = tc::smem_u32(&full[stage]);
          const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
          if (j < mA * kA) {  // phase A: gate + up rows of slice m, token tile
            const int m = j / kA, kb = j - m * kA;
            tc::mbar_arrive_expect_tx(fb, L::STAGE);
            tc::tma_load_2d(sa, &p.map_g, fb, kb * fBK, g * p.h + m * 64);
            tc::tma_load_2d(sa + L::A_BYTES / 2, &p.map_u, fb, kb * fBK, g * p.h + m * 64);
            tc::tma_load_2d(sa + L::A_BYTES, &p.map_x, fb, kb * fBK, tok0);
          } else {  // phase B: 128 down rows of output slice m2
            const int jj = j - mA * kA, m2 = jj / kB, kb = jj - m2 * kB;
            tc::mbar_arrive_expect_tx(fb, L::A_BYTES);
            tc::tma_load_2d(sa, &p.map_d, fb, kb * fBK, g * p.width + m2 * fBM);
          }
          if (++stage == fS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      for (int i = 0; i < fS; ++i) {  // drain loads still in flight
        if (--stage < 0) {
          stage = fS - 1;
          phase ^= 1u;
        }
        tc::mbar_wait(tc::smem_u32(&full[stage]), phase, nullptr, fWaitBudget / 8);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      const uint32_t hs_addr = tc::smem_u32(hs);
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
        int g, n;
        decode(tile, g, n);
        const int n_valid = min(fBN, grp_cnt[g] - n * fBN);
        const uint32_t idesc = tc::idesc_bf16_f32(fBM, (uint32_t)((n_valid + 15) & ~15));
        const uint32_t par = (uint32_t)(it & 1);
        // phase A (its TMEM region was read by the previous tile's epilogue A,
        // which finished before that tile's h_ready)
        for (int m = 0; m < mA && ok; ++m) {
          for (int kb = 0; kb < kA; ++kb) {
            if (!tc::mbar_wait(tc::smem_u32(&full[stage]), phase, abort_flag, fWaitBudget)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
#pragma unroll
            for (int k = 0; k < fBK / 16; ++k)
              tc::mma_bf16(tmem_base + (uint32_t)(m * fBN), tc::smem_desc_sw128(sa + k * 32),
                           tc::smem_desc_sw128(sa + L::A_BYTES + k * 32), idesc,
                           (kb | k) != 0 ? 1u : 0u);
            tc::mma_commit(tc::smem_u32(&empty[stage]));
            if (++stage == fS) {
              stage = 0;
              phase ^= 1u;
            }
          }
          // slice m's accumulator: its epilogue overlaps the next slice's MMAs
          if (ok) tc::mma_commit(tc::smem_u32(&a_done[m]));
        }
        if (!ok) break;
        if (!tc::mbar_wait(tc::smem_u32(h_ready), par, abort_flag, fWaitBudget) ||
            !tc::mbar_wait(tc::smem_u32(b_free), par ^ 1u, abort_flag, fWaitBudget)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        for (int m2 = 0; m2 < mB && ok; ++m2) {
          for (int kb = 0; kb < kB; ++kb) {
            if (!tc::mbar_wait(tc::smem_u32(&full[stage]), phase, abort_flag, fWaitBudget)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
            const uint32_t hb = hs_addr + (uint32_t)(kb * fBN * 128);
#pragma unroll
            for (int k = 0; k < fBK / 16; ++k)
              tc::mma_bf16(tmem_base + (uint32_t)((mA + m2) * fBN),
                           tc::smem_desc_sw128(sa + k * 32), tc::smem_desc_sw128(hb + k * 32),
                           idesc, (kb | k) != 0 ? 1u : 0u);
            tc::mma_commit(tc::smem_u32(&empty[stage]));
            if (++stage == fS) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (ok) tc::mma_commit(tc::smem_u32(&b_done[m2]));
        }
        if (!ok) break;
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        tc::mma_commit(tc::smem_u32(drain));
        tc::mbar_wait(tc::smem_u32(drain), 0, nullptr, fWaitBudget / 8);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, row = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      int g, n;
      decode(tile, g, n);
      const int n_valid = min(fBN, grp_cnt[g] - n * fBN);
      const int tok0 = grp_beg[g] + n * fBN;
      const uint32_t par = (uint32_t)(it & 1);
      bool ok = true;
      // the tile's combine weights, fetched while phase A runs, once every
      // epilogue warp is done with the previous tile's (the named barriers
      // of epilogue A publish them before epilogue B reads them)
      if (p.row_w) {
        asm volatile("bar.sync 1, 128;" ::: "memory");
        for (int i = row; i < fBN; i += 128) fac[i] = i < n_valid ? p.row_w[tok0 + i] : 1.0f;
      }
      // H = act(gate, up) -> bf16 into the swizzled K-major tile (k-block m)
      for (int m = 0; m < mA && ok; ++m) {
        if (!all_epi_ok(tc::mbar_wait(tc::smem_u32(&a_done[m]), par, abort_flag, fWaitBudget))) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        for (int c = 0; c < fBN; c += 32) {
          float v[32];
          tc::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(m * fBN + c),
                                 v);
#pragma unroll
          for (int j = 0; j < 32; ++j) epi[row * fEpiLd + j] = v[j];
          asm volatile("bar.sync 1, 128;" ::: "memory");
          const int tok = c + lane;  // token row of the H tile
          uint32_t packed[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float h0 = gated_act<ACT>(epi[(q * 16 + i) * fEpiLd + lane],
                                            epi[(64 + q * 16 + i) * fEpiLd + lane], p.beta_g,
                                            p.beta_u);
            const float h1 = gated_act<ACT>(epi[(q * 16 + i + 1) * fEpiLd + lane],
                                            epi[(64 + q * 16 + i + 1) * fEpiLd + lane], p.beta_g,
                                            p.beta_u);
            __nv_bfloat162 hv = __floats2bfloat162_rn(h0, h1);
            packed[i >> 1] = *reinterpret_cast<uint32_t*>(&hv);
          }
          // 16-byte chunks 2q and 2q+1 of row `tok`, swizzled by (tok mod 8)
          uint8_t* rowp = hs + m * (fBN * 128) + tok * 128;
          *reinterpret_cast<uint4*>(rowp + (((2 * q) ^ (tok & 7)) << 4)) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
          *reinterpret_cast<uint4*>(rowp + (((2 * q + 1) ^ (tok & 7)) << 4)) =
              make_uint4(packed[4], packed[5], packed[6], packed[7]);
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      // make the generic-proxy stores visible to the tensor core, then hand over
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(h_ready));
      for (int m2 = 0; m2 < mB; ++m2) {
        // output slice m2's accumulator: stored while later slices' MMAs run
        if (!all_epi_ok(tc::mbar_wait(tc::smem_u32(&b_done[m2]), par, abort_flag, fWaitBudget))) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const int col = m2 * fBM + row;
        for (int c = 0; c < n_valid; c += 32) {
          float v[32];
          tc::tmem_ld_32x32b_x32(
              tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((mA + m2) * fBN + c), v);
          // F(u), or a * F(u) when row_w is set (the combine then only adds
          // rows); the weights were staged in shared memory at the tile start.
          // All 32 weights are read before the chunk's first store: a read
          // between stores through generic pointers would wait out its
          // shared-memory latency once per store.
          if (p.row_w) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= fac[c + j];
          }
          float* yf = static_cast<float*>(p.y_rows);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c + j < n_valid) yf[(size_t)(tok0 + c + j) * p.width + col] = v[j];
        }
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(b_free));
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, 512);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)fBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

constexpr size_t fSmemLimit = 227 * 1024;

bool ffn_fused_ok(int width, int h, int G) {
  return h % 64 == 0 && h <= fHMax && width % fBM == 0 && width >= fBM &&
         (h / 64 + width / fBM) * fBN <= 512 && FLayout::bytes(G) <= fSmemLimit;
}

int launch_ffn_fused(int G, int64_t R, int width, int h, const __nv_bfloat16* x_rows,
                     const int32_t* offsets, const __nv_bfloat16* w_gate,
                     const __nv_bfloat16* w_up, const __nv_bfloat16* w_down, const moe_act& act,
                     void* y_rows, cudaStream_t st, const float* row_w) {
  if (R == 0) return MOE_OK;
  FusedParams p{};
  if (!make_map(&p.map_g, w_gate, (uint64_t)G * h, width, 64) ||
      !make_map(&p.map_u, w_up, (uint64_t)G * h, width, 64) ||
      !make_map(&p.map_x, x_rows, R, width, fBN) ||
      !make_map(&p.map_d, w_down, (uint64_t)G * width, h, fBM))
    return MOE_ERR_CUDA;
  p.offsets = offsets;
  p.R = (int)R;
  p.G = G;
  p.width = width;
  p.h = h;
  p.beta_g = act.beta_gate;
  p.beta_u = act.beta_up;
  p.y_rows = y_rows;
  p.row_w = row_w;
  p.status = status_word();
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(tc_fused_ffn<MOE_ACT_SWIGLU>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)fSmemLimit) != cudaSuccess ||
        cudaFuncSetAttribute(tc_fused_ffn<MOE_ACT_SITU_GLU>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)fSmemLimit) != cudaSuccess)
      return MOE_ERR_CUDA;
    configured[dev] = true;
  }
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (R + fBN - 1) / fBN + G;  // upper bound on the tiles
  if (grid > sms) grid = sms;
  if (act.kind == MOE_ACT_SITU_GLU) {
    MOE_PREFER_SHARED((tc_fused_ffn<MOE_ACT_SITU_GLU>));
    launch_pdl(tc_fused_ffn<MOE_ACT_SITU_GLU>, dim3((unsigned)grid), dim3(fThreads),
               FLayout::bytes(G), st, p);
  } else {
    MOE_PREFER_SHARED((tc_fused_ffn<MOE_ACT_SWIGLU>));
    launch_pdl(tc_fused_ffn<MOE_ACT_SWIGLU>, dim3((unsigned)grid), dim3(fThreads),
               FLayout::bytes(G), st, p);
  }
  return launch_status();
}

}  // namespace moe
