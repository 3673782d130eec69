// Backward GEMMs of the grouped SwiGLU experts on the sm_100a tensor cores
// (tcgen05 + TMEM + TMA), for the layer backward of the tutorial "Mixture of
// Experts MoE: how sparse activation saves compute" (§3.1 expert F, §3.2
// y = sum a F, §3.7 the router term) with the selected sets held fixed.
//
// The backward contracts the forward's operands along their other dimension,
// so the weights and the activation rows are read MN-major (the M or N index
// contiguous in memory) instead of being transposed in HBM:
//   dgrad  (A = a weight matrix read MN-major, B = token rows K-major)
//     dH'  = dy W_down          per expert, K = d; epilogue: with the saved
//            pre-activations g, v and the combine weight a, it forms
//            dg = a dH' v' SiLU'(g') J_g, dv = a dH' SiLU(g') J_v (bf16) and
//            the per-tile partial sums of dH' . H for da = dy . F
//     dX   = dG W_gate + dV W_up   K = h, two K-segments, fp32 rows
//   wgrad  (A and B both token rows read MN-major, K = the expert's rows)
//     dW_gate = dG^T X, dW_up = dV^T X, dW_down = (a dy)^T H   fp32
// Row ranges are padded to multiples of 64 per expert with zero rows, so a
// K-block never reaches into the next expert's rows.
//
// Same structure as the forward kernel: persistent CTAs, one TMA producer
// thread, one MMA thread, four epilogue warps, two TMEM accumulators, bounded
// mbarrier waits (MOE_ERR_TIMEOUT, drain, TMEM freed).
#include <cuda.h>

#include "common.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace {

constexpr int wBM = 128, wBK = 64, wBN = 128, wS = 6, wThreads = 192, wEpiLd = 33;
constexpr long long wWaitBudget = 4000000000LL;

struct BwdParams {
  CUtensorMap maps[4];
  const int32_t* offsets;  // [G+1] padded row ranges (multiples of 64)
  int rows;                // rows of the token-row operands and outputs
  int G;
  int nseg;
  int seg_end[2];          // cumulative k-blocks (dgrad)
  int amap[2], bmap[2];
  int a_krow[2];           // dgrad: K row offset of A inside a group
  int b_col[2];            // dgrad: column offset of B
  int a_k_per_group;       // dgrad: K rows of A owned by one group
  int m_tiles, n_tiles;    // M tiles; wgrad: N tiles per group
  int mode;
  int act_kind;
  float beta_g, beta_u;
  // BWD_ACT
  const __nv_bfloat16* g_pre;  // [rows][h] saved gate pre-activations
  const __nv_bfloat16* v_pre;  // [rows][h] saved up pre-activations
  const float* row_w;          // [rows] combine weight of each row
  int h;
  __nv_bfloat16* dG;           // [rows][h]
  __nv_bfloat16* dV;           // [rows][h]
  float* da_part;              // [rows][m_tiles]
  // DGRAD_F32 / WGRAD_F32
  float* out;
  int out_ld;
  int64_t out_group_stride;    // wgrad: elements per group's matrix
  int* status;
};

enum { BMODE_ACT = 0, BMODE_DGRAD_F32 = 1, BMODE_WGRAD_F32 = 2 };

struct WLayout {
  static constexpr int A_BYTES = wBM * wBK * 2;
  static constexpr int B_BYTES = wBN * wBK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = wBM * wEpiLd * 4;
  static size_t bytes(int G) {
    size_t b = 1024 + (size_t)wS * STAGE + EPI_BYTES + (size_t)3 * (G + 1) * 4;
    b = align_up(b, 8);
    b += (size_t)(2 * wS + 5) * 8 + 16;
    return b;
  }
};

__device__ __forceinline__ void named_sync_w() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// MN-major operand tile of 64-element (128-byte) columns: 8 K rows per
// swizzle atom (1024 B, SBO), successive 64-wide MN atoms 8 KB apart (LBO,
// each a 64 x 64 TMA box).  Fields as in smem_desc_sw128.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(8192 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16, bf16 A and B, fp32 D, A MN-major (bit 15), B MN-major (bit 16)
// when b_mn.
__device__ __forceinline__ uint32_t idesc_bwd(uint32_t N, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((N >> 3) << 17) | ((uint32_t)(wBM >> 4) << 24);
}

template <int ACT, bool WGRAD>
__global__ void __launch_bounds__(wThreads, 1) tc_bwd_gemm(const __grid_constant__ BwdParams p) {
  using L = WLayout;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  float* epi = reinterpret_cast<float*>(smem + wS * L::STAGE);
  int* grp_beg = reinterpret_cast<int*>(epi + wBM * wEpiLd);
  int* grp_cnt = grp_beg + (p.G + 1);
  int* grp_pre = grp_cnt + (p.G + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(grp_pre + p.G + 1) + 7) & ~static_cast<uintptr_t>(7));
  uint64_t* full = bars;
  uint64_t* empty = bars + wS;
  uint64_t* tfull = bars + 2 * wS;
  uint64_t* tempty = bars + 2 * wS + 2;
  uint64_t* drain = bars + 2 * wS + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * wS + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int s = 0; s < wS; ++s) {
      tc::mbar_init(tc::smem_u32(&full[s]), 1);
      tc::mbar_init(tc::smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(tc::smem_u32(&tfull[b]), 1);
      tc::mbar_init(tc::smem_u32(&tempty[b]), 128);
    }
    tc::mbar_init(tc::smem_u32(drain), 1);
    tc::fence_barrier_init();
    for (int i = 0; i < 4; ++i) tc::tma_prefetch_desc(&p.maps[i]);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 2 * wBN);
    tc::tmem_relinquish();
  }
  pdl_wait();
  pdl_allow_next();

  // group table: row range and tile prefix per group
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int g = base + lane;
      int beg = 0, cnt = 0;
      if (g < p.G) {
        beg = p.offsets[g];
        cnt = p.offsets[g + 1] - beg;
        if (cnt < 0 || beg < 0 || (cnt & 63) != 0 || beg > p.rows || cnt > p.rows - beg) {
          record_error(p.status, MOE_ERR_BOUNDS);
          cnt = (cnt < 0 || beg < 0 || beg > p.rows || cnt > p.rows - beg) ? 0 : cnt & ~63;
        }
      }
      int t = 0;
      if (g < p.G) t = WGRAD ? p.m_tiles * p.n_tiles : p.m_tiles * ((cnt + wBN - 1) / wBN);
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

  auto decode = [&](int tile, int& g, int& m, int& n) {
    int lo = 0, hi = p.G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (grp_pre[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
    const int local = tile - grp_pre[g];
    const int nt = WGRAD ? p.n_tiles : (grp_cnt[g] + wBN - 1) / wBN;
    m = local / nt;
    n = local - m * nt;
  };
  // k-blocks of a tile: the fixed reduction of dgrad, the group's rows / 64 of wgrad
  auto kblocks_of = [&](int g) { return WGRAD ? grp_cnt[g] / wBK : p.seg_end[p.nseg - 1]; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int g, m, n;
        decode(tile, g, m, n);
        const int kbs = kblocks_of(g);
        int seg = 0, seg_start = 0;
        for (int kb = 0; kb < kbs; ++kb) {
          if (!WGRAD)
            while (kb >= p.seg_end[seg]) seg_start = p.seg_end[seg++];
          if (!tc::mbar_wait(tc::smem_u32(&empty[stage]), phase ^ 1u, abort_flag, wWaitBudget)) {
            ok = false;
            break;
          }
          const uint32_t fb = tc::smem_u32(&full[stage]);
          tc::mbar_arrive_expect_tx(fb, L::STAGE);
          const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
          const uint32_t sb = sa + L::A_BYTES;
          if (WGRAD) {
            // both operands: 64 x 64 boxes (features inner) of the group's rows
            const int y = grp_beg[g] + kb * wBK;
            tc::tma_load_2d(sa, &p.maps[0], fb, m * wBM, y);
            tc::tma_load_2d(sa + 8192, &p.maps[0], fb, m * wBM + 64, y);
            tc::tma_load_2d(sb, &p.maps[1], fb, n * wBN, y);
            tc::tma_load_2d(sb + 8192, &p.maps[1], fb, n * wBN + 64, y);
          } else {
            // A: the group's weight matrix read MN-major; B: token rows K-major
            const int kx = (kb - seg_start) * wBK;
            const int ay = g * p.a_k_per_group + p.a_krow[seg] + kx;
            tc::tma_load_2d(sa, &p.maps[p.amap[seg]], fb, m * wBM, ay);
            tc::tma_load_2d(sa + 8192, &p.maps[p.amap[seg]], fb, m * wBM + 64, ay);
            tc::tma_load_2d(sb, &p.maps[p.bmap[seg]], fb, p.b_col[seg] + kx,
                            grp_beg[g] + n * wBN);
          }
          if (++stage == wS) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      for (int i = 0; i < wS; ++i) {
        if (--stage < 0) {
          stage = wS - 1;
          phase ^= 1u;
        }
        tc::mbar_wait(tc::smem_u32(&full[stage]), phase, nullptr, wWaitBudget / 8);
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
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
        int g, m, n;
        decode(tile, g, m, n);
        const int kbs = kblocks_of(g);
        const int n_valid = WGRAD ? wBN : min(wBN, grp_cnt[g] - n * wBN);
        const uint32_t idesc = idesc_bwd((uint32_t)((n_valid + 15) & ~15), WGRAD);
        const int b = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!tc::mbar_wait(tc::smem_u32(&tempty[b]), (use & 1u) ^ 1u, abort_flag, wWaitBudget)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(b * wBN);
        for (int kb = 0; kb < kbs; ++kb) {
          if (!tc::mbar_wait(tc::smem_u32(&full[stage]), phase, abort_flag, wWaitBudget)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
          const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
          for (int k = 0; k < wBK / 16; ++k) {
            // MN-major: 16 K rows = two 8-row atoms = 2048 bytes per step
            const uint64_t ad = smem_desc_mn_sw128(sa + k * 2048);
            const uint64_t bd = WGRAD ? smem_desc_mn_sw128(sb + k * 2048)
                                      : tc::smem_desc_sw128(sb + k * 32);
            tc::mma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc::mma_commit(tc::smem_u32(&empty[stage]));
          if (++stage == wS) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::mma_commit(tc::smem_u32(&tfull[b]));  // also with no k-block (empty group)
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        tc::mma_commit(tc::smem_u32(drain));
        tc::mbar_wait(tc::smem_u32(drain), 0, nullptr, wWaitBudget / 8);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      int g, m, n;
      decode(tile, g, m, n);
      const int n_valid = WGRAD ? wBN : min(wBN, grp_cnt[g] - n * wBN);
      const int tok0 = grp_beg[g] + n * wBN;
      const bool empty_group = kblocks_of(g) == 0;
      const int b = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      const bool got = tc::mbar_wait(tc::smem_u32(&tfull[b]), use & 1u, abort_flag, wWaitBudget);
      uint32_t all_ok;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\t"
          "setp.ne.u32 p, %1, 0;\n\t"
          "bar.red.and.pred q, 1, 128, p;\n\t"
          "selp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(all_ok)
          : "r"((uint32_t)got)
          : "memory");
      if (!all_ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc::tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * wBN);
      for (int c = 0; c < n_valid; c += 32) {
        float v[32];
        tc::tmem_ld_32x32b_x32(t_row + (uint32_t)c, v);
        if (WGRAD) {
          // dW[g][m*128 + row][n*128 + c .. c+31], zero for an expert with no rows
          float* o = p.out + (size_t)g * p.out_group_stride +
                     (size_t)(m * wBM + row) * p.out_ld + n * wBN + c;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(o + j) =
                empty_group ? make_float4(0.f, 0.f, 0.f, 0.f)
                            : make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        } else if (p.mode == BMODE_DGRAD_F32) {
          const int col = m * wBM + row;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c + j < n_valid) p.out[(size_t)(tok0 + c + j) * p.out_ld + col] = v[j];
        } else {
          // dH'[r][j] for hidden unit j = m*128 + row and rows r = tok0 + c + jj
          const int hj = m * wBM + row;
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            float hterm = 0.0f;
            if (c + jj < n_valid) {
              const size_t r = (size_t)(tok0 + c + jj);
              const float g0 = __bfloat162float(p.g_pre[r * p.h + hj]);
              const float v0 = __bfloat162float(p.v_pre[r * p.h + hj]);
              const float a = p.row_w[r];
              float gc = g0, vc = v0, jg = 1.0f, jv = 1.0f;
              if (ACT == MOE_ACT_SITU_GLU) {
                const float tg = tanhf(g0 / p.beta_g), tv = tanhf(v0 / p.beta_u);
                gc = p.beta_g * tg;
                vc = p.beta_u * tv;
                jg = 1.0f - tg * tg;
                jv = 1.0f - tv * tv;
              }
              const float sg = 1.0f / (1.0f + expf(-gc));
              const float silu = gc * sg;
              const float dh = v[jj];
              p.dG[r * p.h + hj] =
                  __float2bfloat16_rn(a * dh * vc * (sg * (1.0f + gc * (1.0f - sg))) * jg);
              p.dV[r * p.h + hj] = __float2bfloat16_rn(a * dh * silu * jv);
              hterm = dh * silu * vc;  // dH' . H for this unit
            }
            epi[row * wEpiLd + jj] = hterm;
          }
          named_sync_w();
          // per row r: the sum over this tile's 128 hidden units, fixed order
          if (row < 32 && c + row < n_valid) {
            float acc = 0.0f;
            for (int i = 0; i < wBM; ++i) acc += epi[i * wEpiLd + row];
            p.da_part[(size_t)(tok0 + c + row) * p.m_tiles + m] = acc;
          }
          named_sync_w();
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(tc::smem_u32(&tempty[b]));
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, 2 * wBN);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// bf16 [rows][cols], box 64 (columns) x box_rows, 128-byte swizzle.
bool make_bmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_rows) {
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
  cuuint32_t box[2] = {64u, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int ACT, bool WGRAD>
int launch_bwd(const BwdParams& p, int64_t tiles_upper, cudaStream_t st) {
  auto kernel = tc_bwd_gemm<ACT, WGRAD>;
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || !device_slot(dev)) return MOE_ERR_CUDA;
  if (needs_setup(configured, dev)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)WLayout::bytes(1024)) != cudaSuccess)
      return MOE_ERR_CUDA;
    mark_setup(configured, dev);
  }
  MOE_PREFER_SHARED((tc_bwd_gemm<ACT, WGRAD>));
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = sms > 0 ? sms : 148;
  if (tiles_upper < grid) grid = tiles_upper;
  if (grid <= 0) return MOE_OK;
  launch_pdl(kernel, dim3((unsigned)grid), dim3(wThreads), WLayout::bytes(p.G), st, p);
  return launch_status();
}

}  // namespace

// dH' = dy_rows W_down per group (K = width), epilogue forming dG, dV and the
// da partials (see the file comment).  rows: padded row count; offsets: the
// padded group ranges.
int bwd_dgrad_act(const int32_t* offsets, int G, int64_t rows, int width, int h,
                  const __nv_bfloat16* dy_rows, const __nv_bfloat16* w_down,
                  const __nv_bfloat16* g_pre, const __nv_bfloat16* v_pre, const float* row_w,
                  const moe_act& act, __nv_bfloat16* dG, __nv_bfloat16* dV, float* da_part,
                  cudaStream_t st) {
  if (h % wBM != 0 || width % wBK != 0) return MOE_ERR_UNSUPPORTED;
  BwdParams p{};
  // A: W_down [G*width][h] read MN-major (h contiguous), K = width rows per group
  if (!make_bmap(&p.maps[0], w_down, (uint64_t)G * width, h, 64) ||
      !make_bmap(&p.maps[1], dy_rows, rows, width, wBN))
    return MOE_ERR_CUDA;
  p.maps[2] = p.maps[3] = p.maps[0];
  p.offsets = offsets;
  p.rows = (int)rows;
  p.G = G;
  p.nseg = 1;
  p.seg_end[0] = width / wBK;
  p.amap[0] = 0;
  p.bmap[0] = 1;
  p.a_k_per_group = width;
  p.m_tiles = h / wBM;
  p.mode = BMODE_ACT;
  p.act_kind = act.kind;
  p.beta_g = act.beta_gate;
  p.beta_u = act.beta_up;
  p.g_pre = g_pre;
  p.v_pre = v_pre;
  p.row_w = row_w;
  p.h = h;
  p.dG = dG;
  p.dV = dV;
  p.da_part = da_part;
  p.status = status_word();
  const int64_t upper = (int64_t)p.m_tiles * ((rows + wBN - 1) / wBN + G);
  return act.kind == MOE_ACT_SITU_GLU ? launch_bwd<MOE_ACT_SITU_GLU, false>(p, upper, st)
                                      : launch_bwd<MOE_ACT_SWIGLU, false>(p, upper, st);
}

// dX = dG W_gate + dV W_up per group (K = h, two segments), fp32 [rows][width].
int bwd_dgrad_x(const int32_t* offsets, int G, int64_t rows, int width, int h,
                const __nv_bfloat16* dG, const __nv_bfloat16* dV, const __nv_bfloat16* w_gate,
                const __nv_bfloat16* w_up, float* dX, cudaStream_t st) {
  if (h % wBK != 0 || width % wBM != 0) return MOE_ERR_UNSUPPORTED;
  BwdParams p{};
  // A: W_gate, W_up [G*h][width] read MN-major (width contiguous), K = h rows per group
  if (!make_bmap(&p.maps[0], w_gate, (uint64_t)G * h, width, 64) ||
      !make_bmap(&p.maps[1], w_up, (uint64_t)G * h, width, 64) ||
      !make_bmap(&p.maps[2], dG, rows, h, wBN) || !make_bmap(&p.maps[3], dV, rows, h, wBN))
    return MOE_ERR_CUDA;
  p.offsets = offsets;
  p.rows = (int)rows;
  p.G = G;
  p.nseg = 2;
  p.seg_end[0] = h / wBK;
  p.seg_end[1] = 2 * h / wBK;
  p.amap[0] = 0;
  p.amap[1] = 1;
  p.bmap[0] = 2;
  p.bmap[1] = 3;
  p.a_k_per_group = h;
  p.m_tiles = width / wBM;
  p.mode = BMODE_DGRAD_F32;
  p.out = dX;
  p.out_ld = width;
  p.status = status_word();
  const int64_t upper = (int64_t)p.m_tiles * ((rows + wBN - 1) / wBN + G);
  return launch_bwd<MOE_ACT_SWIGLU, false>(p, upper, st);
}

// out [rows][M] fp32 = B [rows][K] A_g, A [G*K][M] read MN-major: one K-segment
// of the dgrad GEMM with the plain fp32 epilogue (dense layers use G = 1).
int bwd_dgrad_plain(const int32_t* offsets, int G, int64_t rows, int K, int M,
                    const __nv_bfloat16* B, const __nv_bfloat16* A, float* out,
                    cudaStream_t st) {
  if (K % wBK != 0 || M % wBM != 0) return MOE_ERR_UNSUPPORTED;
  BwdParams p{};
  if (!make_bmap(&p.maps[0], A, (uint64_t)G * K, M, 64) ||
      !make_bmap(&p.maps[1], B, rows, K, wBN))
    return MOE_ERR_CUDA;
  p.maps[2] = p.maps[3] = p.maps[0];
  p.offsets = offsets;
  p.rows = (int)rows;
  p.G = G;
  p.nseg = 1;
  p.seg_end[0] = K / wBK;
  p.amap[0] = 0;
  p.bmap[0] = 1;
  p.a_k_per_group = K;
  p.m_tiles = M / wBM;
  p.mode = BMODE_DGRAD_F32;
  p.out = out;
  p.out_ld = M;
  p.status = status_word();
  const int64_t upper = (int64_t)p.m_tiles * ((rows + wBN - 1) / wBN + G);
  return launch_bwd<MOE_ACT_SWIGLU, false>(p, upper, st);
}

// dW[g] = A_g^T B_g over group g's rows: A [rows][M] and B [rows][Ncols]
// read MN-major; dW fp32 [G][M][Ncols].
int bwd_wgrad(const int32_t* offsets, int G, int64_t rows, const __nv_bfloat16* A, int M,
              const __nv_bfloat16* B, int Ncols, float* dW, cudaStream_t st) {
  if (M % wBM != 0 || Ncols % wBN != 0) return MOE_ERR_UNSUPPORTED;
  BwdParams p{};
  if (!make_bmap(&p.maps[0], A, rows, M, 64) || !make_bmap(&p.maps[1], B, rows, Ncols, 64))
    return MOE_ERR_CUDA;
  p.maps[2] = p.maps[3] = p.maps[0];
  p.offsets = offsets;
  p.rows = (int)rows;
  p.G = G;
  p.nseg = 1;
  p.m_tiles = M / wBM;
  p.n_tiles = Ncols / wBN;
  p.mode = BMODE_WGRAD_F32;
  p.out = dW;
  p.out_ld = Ncols;
  p.out_group_stride = (int64_t)M * Ncols;
  p.status = status_word();
  const int64_t upper = (int64_t)G * p.m_tiles * p.n_tiles;
  return launch_bwd<MOE_ACT_SWIGLU, true>(p, upper, st);
}

}  // namespace moe
