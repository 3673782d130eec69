// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Tutorial "Mixture of Experts MoE: how sparse activation saves compute",
// §3.1 equation F and §3.6 (expert i works on its own [L_i, d] rows):
//   gate/up:  H = act(X_e W_gate,e^T, X_e W_up,e^T)   -> bf16 [rows][h]
//   down:     Y = H_e W_down,e^T                       -> fp32 [rows][width]
//
// Orientation: the expert WEIGHTS are the MMA's M operand (128 rows per tile)
// and the expert's TOKENS are its N operand (up to BN per tile, rounded up to
// 16), so a ragged last token tile of an expert costs only its own columns.
// For gate/up the 128 weight rows of a tile are 64 gate rows stacked on the
// 64 matching up rows (two TMA boxes), so one accumulator holds both halves
// and the epilogue applies SiLU(g) * u (or the SiTU-GLU soft caps of the
// Stable LatentMoE document) and stores bf16 H.
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0    TMA producer (one elected lane), S-stage smem ring
//   warp 1    TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-5 epilogue: tcgen05.ld TMEM -> registers -> global
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap
// the MMAs of tile i+1.  Every mbarrier wait is bounded; a wait that runs out
// records MOE_ERR_TIMEOUT, stops all roles, drains in-flight TMA loads and
// frees TMEM before the CTA exits.
#include <cuda.h>

#include "common.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 bf16 = 128 bytes = one swizzle span
constexpr int kThreads = 192;
constexpr long long kWaitBudget = 4000000000LL;  // cycles (~2 s)
constexpr int kEpiLd = 33;                       // padded row of the gate/up exchange tile


constexpr int kMaxSeg = 3;

// One GEMM problem.  The reduction runs over up to kMaxSeg K-segments that
// accumulate into the same tile; segment s reads A from maps[amap[s]] (rows
// offset by arow[s]) and B from maps[bmap[s]] (columns offset by bcol[s]).
// Gate/up mode has one segment: A rows 0-63 from maps[0] (gate), rows 64-127
// from maps[1] (up), B from maps[2].
struct TcParams {
  CUtensorMap maps[4];
  const int32_t* offsets;  // [G+1] token row ranges; nullptr: every group uses rows [0, T)
  int T;
  int G;
  int nseg;
  int seg_end[kMaxSeg];   // cumulative 64-wide k-blocks at the end of each segment
  int amap[kMaxSeg], bmap[kMaxSeg];
  int arow[kMaxSeg], bcol[kMaxSeg];
  int a_rows_per_group;   // rows of A owned by one group
  int m_tiles;            // 128-row tiles of A per group
  int mode;
  int act_kind;
  float beta_g, beta_u;
  void* out;
  int out_ld;             // elements per output row
  int out_col_group;      // output column offset per group (groups sharing tokens)
  int* status;
};

__device__ __forceinline__ void named_sync_epi() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int BN, int S>
struct Layout {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = kBM * kEpiLd * 4;
  static size_t bytes(int G) {
    size_t b = 1024;  // alignment slack of the dynamic smem base
    b += (size_t)S * STAGE + EPI_BYTES;
    b += (size_t)3 * (G + 1) * 4;
    b = align_up(b, 8);
    b += (size_t)(2 * S + 5) * 8 + 16;
    return b;
  }
};

template <int BN, int S, int ACT>
__global__ void __launch_bounds__(kThreads, 1) tc_grouped_gemm(const __grid_constant__ TcParams p) {
  using L = Layout<BN, S>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  float* epi = reinterpret_cast<float*>(smem + S * L::STAGE);
  int* grp_beg = reinterpret_cast<int*>(epi + kBM * kEpiLd);
  int* grp_cnt = grp_beg + (p.G + 1);
  int* grp_pre = grp_cnt + (p.G + 1);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(grp_pre + p.G + 1) + 7) & ~static_cast<uintptr_t>(7));
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* drain = bars + 2 * S + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool fused = p.mode == MODE_GATEUP;

  // ---- prologue that reads no data of the previous kernel: barriers, TMEM,
  // tensor-map prefetch; it overlaps the previous kernel's tail (PDL)
  if (warp == 0 && lane == 0) {
    *abort_flag = 0;
    for (int s = 0; s < S; ++s) {
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
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 2 * BN);
    tc::tmem_relinquish();
  }
  pdl_wait();
  pdl_allow_next();

  // ---- group table: token range and tile prefix per group (warp 0 scans)
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int g = base + lane;
      int beg = 0, cnt = 0;
      if (g < p.G) {
        if (p.offsets) {
          beg = p.offsets[g];
          cnt = p.offsets[g + 1] - beg;
          if (cnt < 0 || beg < 0) {
            record_error(p.status, MOE_ERR_BOUNDS);
            cnt = 0;
          }
        } else {
          cnt = p.T;
        }
      }
      const int t = g < p.G ? p.m_tiles * ((cnt + BN - 1) / BN) : 0;
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
  const int kblocks = p.seg_end[p.nseg - 1];

  auto decode = [&](int tile, int& g, int& m, int& n) {
    int lo = 0, hi = p.G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (grp_pre[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
    const int local = tile - grp_pre[g];
    const int nt = (grp_cnt[g] + BN - 1) / BN;
    m = local / nt;
    n = local - m * nt;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int g, m, n;
        decode(tile, g, m, n);
        const int a_row = g * p.a_rows_per_group + m * (fused ? 64 : kBM);
        const int b_row = grp_beg[g] + n * BN;
        int seg = 0, seg_start = 0;
        for (int kb = 0; kb < kblocks; ++kb) {
          while (kb >= p.seg_end[seg]) seg_start = p.seg_end[seg++];
          const int kx = (kb - seg_start) * kBK;
          if (!tc::mbar_wait(tc::smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kWaitBudget)) {
            ok = false;
            break;
          }
          const uint32_t fb = tc::smem_u32(&full[stage]);
          tc::mbar_arrive_expect_tx(fb, L::STAGE);
          const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
          const uint32_t sb = sa + L::A_BYTES;
          if (fused) {
            tc::tma_load_2d(sa, &p.maps[0], fb, kx, a_row);
            tc::tma_load_2d(sa + L::A_BYTES / 2, &p.maps[1], fb, kx, a_row);
            tc::tma_load_2d(sb, &p.maps[2], fb, kx, b_row);
          } else {
            tc::tma_load_2d(sa, &p.maps[p.amap[seg]], fb, kx, a_row + p.arow[seg]);
            tc::tma_load_2d(sb, &p.maps[p.bmap[seg]], fb, p.bcol[seg] + kx, b_row);
          }
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      // Drain: the last S issued stages may still have loads in flight.
      for (int i = 0; i < S; ++i) {
        if (--stage < 0) {
          stage = S - 1;
          phase ^= 1u;
        }
        tc::mbar_wait(tc::smem_u32(&full[stage]), phase, nullptr, kWaitBudget / 8);
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
        const int n_valid = min(BN, grp_cnt[g] - n * BN);
        const uint32_t n_mma = (uint32_t)((n_valid + 15) & ~15);
        const uint32_t idesc = tc::idesc_bf16_f32(kBM, n_mma);
        const int b = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!tc::mbar_wait(tc::smem_u32(&tempty[b]), (use & 1u) ^ 1u, abort_flag, kWaitBudget)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait(tc::smem_u32(&full[stage]), phase, abort_flag, kWaitBudget)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
          const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            tc::mma_bf16(d_tmem, tc::smem_desc_sw128(sa + k * 32), tc::smem_desc_sw128(sb + k * 32),
                         idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc::mma_commit(tc::smem_u32(&empty[stage]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::mma_commit(tc::smem_u32(&tfull[b]));
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        // Let every MMA issued so far finish before TMEM is released.
        tc::mma_commit(tc::smem_u32(drain));
        tc::mbar_wait(tc::smem_u32(drain), 0, nullptr, kWaitBudget / 8);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      int g, m, n;
      decode(tile, g, m, n);
      const int n_valid = min(BN, grp_cnt[g] - n * BN);
      const int tok0 = grp_beg[g] + n * BN;
      const int b = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      // The four epilogue warps share named barriers, so they take the
      // give-up decision together.
      const bool got = tc::mbar_wait(tc::smem_u32(&tfull[b]), use & 1u, abort_flag, kWaitBudget);
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
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * BN);
      for (int c = 0; c < n_valid; c += 32) {
        float v[32];
        tc::tmem_ld_32x32b_x32(t_row + (uint32_t)c, v);
        if (p.mode == MODE_GATEUP) {
#pragma unroll
          for (int j = 0; j < 32; ++j) epi[row * kEpiLd + j] = v[j];
          named_sync_epi();
          const int tok = c + lane;
          if (tok < n_valid) {
            uint32_t packed[8];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              const float h0 = gated_act<ACT>(epi[(q * 16 + i) * kEpiLd + lane],
                                              epi[(64 + q * 16 + i) * kEpiLd + lane], p.beta_g,
                                              p.beta_u);
              const float h1 = gated_act<ACT>(epi[(q * 16 + i + 1) * kEpiLd + lane],
                                              epi[(64 + q * 16 + i + 1) * kEpiLd + lane],
                                              p.beta_g, p.beta_u);
              __nv_bfloat162 hv = __floats2bfloat162_rn(h0, h1);
              packed[i >> 1] = *reinterpret_cast<uint32_t*>(&hv);
            }
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) +
                               (size_t)(tok0 + tok) * p.out_ld + g * p.out_col_group + m * 64 +
                               q * 16;
            reinterpret_cast<uint4*>(o)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            reinterpret_cast<uint4*>(o)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
          named_sync_epi();
        } else {
          const int col = g * p.out_col_group + m * kBM + row;
          if (p.mode == MODE_STORE_F32) {
            float* o = static_cast<float*>(p.out);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c + j < n_valid) o[(size_t)(tok0 + c + j) * p.out_ld + col] = v[j];
          } else {
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c + j < n_valid)
                o[(size_t)(tok0 + c + j) * p.out_ld + col] = __float2bfloat16_rn(v[j]);
          }
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
    tc::tmem_dealloc(tmem_base, 2 * BN);
  }
}

// ------------------------------------------------------------------- host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Row-major bf16 matrix [rows][cols] viewed as a 2-D tensor, box 64 x box_rows,
// 128-byte swizzle (the layout smem_desc_sw128 describes).
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!device_slot(dev)) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <int BN, int S, int ACT>
int launch_tc(const TcParams& p, int64_t tiles_upper, cudaStream_t st) {
  const size_t smem = Layout<BN, S>::bytes(p.G);
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (needs_setup(configured, dev)) {
    if (cudaFuncSetAttribute(tc_grouped_gemm<BN, S, ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Layout<BN, S>::bytes(1024)) != cudaSuccess)
      return MOE_ERR_CUDA;
    mark_setup(configured, dev);
  }
  int64_t grid = sm_count();
  if (tiles_upper < grid) grid = tiles_upper;
  if (grid <= 0) return MOE_OK;
  MOE_PREFER_SHARED((tc_grouped_gemm<BN, S, ACT>));
  launch_pdl(tc_grouped_gemm<BN, S, ACT>, dim3((unsigned)grid), dim3(kThreads), smem, st, p);
  return launch_status();
}

// Token tile width: 128 columns when groups average under 192 rows (a
// 256-wide tile would be mostly padding) or when 256-wide tiles would not
// give every SM two tiles; 256 otherwise.
int pick_bn(int m_tiles, int64_t max_rows, int G) {
  if (max_rows < 192LL * G) return 128;
  const int64_t up256 = (int64_t)m_tiles * ((max_rows + 255) / 256 + G);
  return up256 >= 2LL * sm_count() ? 256 : 128;
}

int launch_tc_bn(const TcParams& p, int64_t max_rows, int bn, cudaStream_t st) {
  const int64_t upper = (int64_t)p.m_tiles * ((max_rows + bn - 1) / bn + p.G);
  const bool situ = p.mode == MODE_GATEUP && p.act_kind == MOE_ACT_SITU_GLU;
  if (bn == 256)
    return situ ? launch_tc<256, 4, MOE_ACT_SITU_GLU>(p, upper, st)
                : launch_tc<256, 4, MOE_ACT_SWIGLU>(p, upper, st);
  return situ ? launch_tc<128, 6, MOE_ACT_SITU_GLU>(p, upper, st)
              : launch_tc<128, 6, MOE_ACT_SWIGLU>(p, upper, st);
}

}  // namespace

size_t ffn_tc_ws_bytes(const moe_shape& s, int32_t /*width*/) {
  return align_up((size_t)s.T * s.k * s.h * 2, 256);
}

int launch_ffn_tc(const moe_shape& s, int32_t width, const __nv_bfloat16* x_rows,
                  const int32_t* offsets, const __nv_bfloat16* w_gate, const __nv_bfloat16* w_up,
                  const __nv_bfloat16* w_down, const moe_act& act, float* y_rows, void* ws,
                  cudaStream_t st) {
  const int64_t R = (int64_t)s.T * s.k;
  if (R == 0) return MOE_OK;
  if (ffn_fused_ok(width, s.h, s.N))  // small h: both GEMMs in one launch, H stays on chip
    return launch_ffn_fused(s.N, R, width, s.h, x_rows, offsets, w_gate, w_up, w_down, act,
                            y_rows, st);
  __nv_bfloat16* H = static_cast<__nv_bfloat16*>(ws);
  int rc = tc_gateup(offsets, (int)R, s.N, x_rows, R, width, w_gate, w_up, s.h, act, H, s.h, 0,
                     st);
  if (rc != MOE_OK) return rc;
  TcSeg seg{w_down, (int64_t)s.N * width, s.h, 0, H, R, s.h, 0};
  return tc_store(offsets, (int)R, s.N, width, &seg, 1, y_rows, MODE_STORE_F32, width, st);
}

// Gate/up GEMM with the fused activation: for group g and its rows of X,
// out[row][g * out_col_group + j] = act(X W_gate[g]^T, X W_up[g]^T)[j], bf16.
int tc_gateup(const int32_t* offsets, int T, int G, const __nv_bfloat16* X, int64_t x_rows,
              int K, const __nv_bfloat16* w_gate, const __nv_bfloat16* w_up, int hidden,
              const moe_act& act, __nv_bfloat16* out, int out_ld, int out_col_group,
              cudaStream_t st) {
  TcParams p{};
  const int64_t rows_w = (int64_t)G * hidden;
  const int64_t max_rows = offsets ? x_rows : (int64_t)T * G;
  const int bn = pick_bn(hidden / 64, max_rows, G);
  if (!make_tmap(&p.maps[0], w_gate, rows_w, K, 64) || !make_tmap(&p.maps[1], w_up, rows_w, K, 64) ||
      !make_tmap(&p.maps[2], X, x_rows, K, bn))
    return MOE_ERR_CUDA;
  p.maps[3] = p.maps[2];
  p.offsets = offsets;
  p.T = T;
  p.G = G;
  p.nseg = 1;
  p.seg_end[0] = K / kBK;
  p.a_rows_per_group = hidden;
  p.m_tiles = hidden / 64;
  p.mode = MODE_GATEUP;
  p.act_kind = act.kind;
  p.beta_g = act.beta_gate;
  p.beta_u = act.beta_up;
  p.out = out;
  p.out_ld = out_ld;
  p.out_col_group = out_col_group;
  p.status = status_word();
  return launch_tc_bn(p, max_rows, bn, st);
}

// Plain GEMM over 1..3 K-segments accumulated into one output:
// out[row][g * m_rows + m] = sum_s (A_s[g * a_rows_s + arow_s + m] . B_s[row][bcol_s + ...]).
int tc_store(const int32_t* offsets, int T, int G, int m_rows, const TcSeg* segs, int nseg,
             void* out, int mode, int out_ld, cudaStream_t st) {
  if (nseg < 1 || nseg > kMaxSeg) return MOE_ERR_INVALID_ARG;
  TcParams p{};
  const int64_t max_rows = offsets ? segs[0].b_rows : (int64_t)T * G;
  const int bn = pick_bn(m_rows / kBM, max_rows, G);
  // distinct (pointer, rows, cols, box) tensor maps, at most four
  const void* key_p[4];
  int64_t key_r[4];
  int key_c[4], key_box[4];
  int nmaps = 0;
  auto map_of = [&](const void* ptr, int64_t rows, int cols, int box) -> int {
    for (int i = 0; i < nmaps; ++i)
      if (key_p[i] == ptr && key_r[i] == rows && key_c[i] == cols && key_box[i] == box) return i;
    if (nmaps >= 4) return -1;
    if (!make_tmap(&p.maps[nmaps], ptr, rows, cols, box)) return -2;
    key_p[nmaps] = ptr;
    key_r[nmaps] = rows;
    key_c[nmaps] = cols;
    key_box[nmaps] = box;
    return nmaps++;
  };
  int kb = 0;
  for (int i = 0; i < nseg; ++i) {
    const int ia = map_of(segs[i].a, segs[i].a_rows, segs[i].K, kBM);
    const int ib = map_of(segs[i].b, segs[i].b_rows, segs[i].b_cols, bn);
    if (ia == -1 || ib == -1) return MOE_ERR_UNSUPPORTED;
    if (ia < 0 || ib < 0) return MOE_ERR_CUDA;
    p.amap[i] = ia;
    p.bmap[i] = ib;
    kb += segs[i].K / kBK;
    p.seg_end[i] = kb;
    p.arow[i] = segs[i].arow;
    p.bcol[i] = segs[i].bcol;
  }
  for (int i = nmaps; i < 4; ++i) p.maps[i] = p.maps[0];
  p.offsets = offsets;
  p.T = T;
  p.G = G;
  p.nseg = nseg;
  p.a_rows_per_group = m_rows;
  p.m_tiles = m_rows / kBM;
  p.mode = mode;
  p.out = out;
  p.out_ld = out_ld;
  p.out_col_group = 0;
  p.status = status_word();
  return launch_tc_bn(p, max_rows, bn, st);
}

}  // namespace moe
