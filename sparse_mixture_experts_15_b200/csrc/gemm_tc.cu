// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Tutorial "Mixture of Experts MoE: how sparse activation saves compute",
// §3.1 equation F and §3.6 (expert i works on its own [L_i, d] rows):
//   gate/up:  H = act(X_e W_gate,e^T, X_e W_up,e^T)   -> bf16 [rows][h]
//   down:     Y = H_e W_down,e^T                       -> fp32 [rows][width]
//             (each row times its token's combine weight a in the layer path,
//             so the combine only adds rows)
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
//
// CTA pairs (CG = 2, clusters of two CTAs on neighbouring SMs): one
// tcgen05.mma.cta_group::2 computes a 256 x BN tile.  Each CTA stages its own
// 128 weight rows and its own BN/2 token rows, so a CTA moves 128 + BN/2
// operand rows per k-block instead of 128 + BN for the same MMA work per SM:
// a third less L2 -> shared-memory traffic at BN = 256.  The even CTA issues
// the MMAs and waits for both CTAs' bytes on its own full barriers; each
// MMA completion is multicast to both CTAs' empty barriers; the accumulator
// ready signal goes to both CTAs' epilogues, which each read their 128 TMEM
// lanes and report back to the even CTA.
#include <cuda.h>

#include "common.cuh"
#include "tc_primitives.cuh"

namespace moe {

// SM count of the current device, looked up once per device.
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

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;  // 64 bf16 = 128 bytes = one swizzle span (128 E4M3 codes)
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
  int T;                   // with offsets: rows of B and of the output
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
  // E4M3 operands only: fp32 scale per row of A (gate/up mode: gate rows in
  // a_scale[0], up rows in a_scale[1]); the operand value is
  // scale * e4m3(code).  b_scale (nullable): a factor per row of B, the
  // token rows (E4M3 token scales, or the combine weight a of each grouped
  // row, so the down GEMM stores a * F(u)).
  const float* a_scale[2];
  const float* b_scale;
};

__device__ __forceinline__ void named_sync_epi() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int BN, int S, int CG = 1>
struct Layout {
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN / CG * kBK * 2;  // this CTA's token rows
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = kBM * kEpiLd * 4 + BN * 4;  // exchange tile + token factors
  static size_t bytes(int G) {
    size_t b = 1024;  // alignment slack of the dynamic smem base
    b += (size_t)S * STAGE + EPI_BYTES;
    b += (size_t)3 * (G + 1) * 4;
    b = align_up(b, 8);
    b += (size_t)(2 * S + 5) * 8 + 16;
    return b;
  }
};

// F8: E4M3 A and B (tcgen05 kind::f8f6f4), 128 codes per 128-byte k-block,
// row scales applied in the epilogue; gate/up mode then stores H as E4M3
// codes with no scale.  Otherwise bf16 A and B (kind::f16).
template <int BN, int S, int ACT, int CG, bool F8>
__global__ void __launch_bounds__(kThreads, 1) tc_grouped_gemm(const __grid_constant__ TcParams p) {
  using L = Layout<BN, S, CG>;
  constexpr int KE = F8 ? 2 * kBK : kBK;  // elements per 128-byte k-block
  static_assert(CG == 1 || CG == 2, "one CTA or a CTA pair per MMA");
  // pair geometry: rank 0 issues the MMAs of the pair; tiles are per pair
  const uint32_t rank = CG == 2 ? tc::cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int unit = CG == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = CG == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem;
  float* epi = reinterpret_cast<float*>(smem + S * L::STAGE);
  float* fac = epi + kBM * kEpiLd;  // [BN] the tile's token-row factors (b_scale)
  int* grp_beg = reinterpret_cast<int*>(fac + BN);
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
      // one CTA: every epilogue thread arrives; a pair: one thread per CTA
      // arrives on the even CTA's barrier
      tc::mbar_init(tc::smem_u32(&tempty[b]), CG == 2 ? 2 : 128);
    }
    tc::mbar_init(tc::smem_u32(drain), 1);
    tc::fence_barrier_init();
    for (int i = 0; i < 4; ++i) tc::tma_prefetch_desc(&p.maps[i]);
  }
  if (warp == 1) {
    if (CG == 2) {
      tc::tmem_alloc_pair(tc::smem_u32(tmem_slot), 2 * BN);
      tc::tmem_relinquish_pair();
    } else {
      tc::tmem_alloc(tc::smem_u32(tmem_slot), 2 * BN);
      tc::tmem_relinquish();
    }
  }
  if (CG == 2) {
    // both CTAs' barriers exist before either CTA signals the other's
    tc::tc_fence_before();
    tc::cluster_sync();
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
          if (cnt < 0 || beg < 0 || beg > p.T || cnt > p.T - beg) {  // rows outside the buffers
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

  // n_mma: MMA width of a tile with n_valid token columns (multiple of 16)
  auto mma_width = [&](int n_valid) { return (n_valid + 15) & ~15; };
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
      for (int tile = unit; tile < total_tiles && ok; tile += n_units) {
        int g, m, n;
        decode(tile, g, m, n);
        // this CTA's weight rows: a pair splits a tile's 256 rows 128 / 128
        // (gate/up: 64 + 64 hidden units each) and its tokens n_mma/2 each
        const int a_row = g * p.a_rows_per_group + m * CG * (fused ? 64 : kBM) +
                          (int)rank * (fused ? 64 : kBM);
        const int n_valid = min(BN, grp_cnt[g] - n * BN);
        const int b_row = grp_beg[g] + n * BN + (int)rank * (mma_width(n_valid) / 2);
        int seg = 0, seg_start = 0;
        for (int kb = 0; kb < kblocks; ++kb) {
          while (kb >= p.seg_end[seg]) seg_start = p.seg_end[seg++];
          const int kx = (kb - seg_start) * KE;
          if (!tc::mbar_wait(tc::smem_u32(&empty[stage]), phase ^ 1u, abort_flag, kWaitBudget)) {
            ok = false;
            break;
          }
          const uint32_t sa = tc::smem_u32(stages + stage * L::STAGE);
          const uint32_t sb = sa + L::A_BYTES;
          if (CG == 2) {
            // both CTAs' bytes complete on the even CTA's full barrier
            const uint32_t fb = tc::mapa_shared(tc::smem_u32(&full[stage]), 0u);
            if (leader) tc::mbar_arrive_expect_tx(tc::smem_u32(&full[stage]), 2 * L::STAGE);
            if (fused) {
              tc::tma_load_2d_pair(sa, &p.maps[0], fb, kx, a_row);
              tc::tma_load_2d_pair(sa + L::A_BYTES / 2, &p.maps[1], fb, kx, a_row);
              tc::tma_load_2d_pair(sb, &p.maps[2], fb, kx, b_row);
            } else {
              tc::tma_load_2d_pair(sa, &p.maps[p.amap[seg]], fb, kx, a_row + p.arow[seg]);
              tc::tma_load_2d_pair(sb, &p.maps[p.bmap[seg]], fb, p.bcol[seg] + kx, b_row);
            }
          } else {
            const uint32_t fb = tc::smem_u32(&full[stage]);
            tc::mbar_arrive_expect_tx(fb, L::STAGE);
            if (fused) {
              tc::tma_load_2d(sa, &p.maps[0], fb, kx, a_row);
              tc::tma_load_2d(sa + L::A_BYTES / 2, &p.maps[1], fb, kx, a_row);
              tc::tma_load_2d(sb, &p.maps[2], fb, kx, b_row);
            } else {
              tc::tma_load_2d(sa, &p.maps[p.amap[seg]], fb, kx, a_row + p.arow[seg]);
              tc::tma_load_2d(sb, &p.maps[p.bmap[seg]], fb, p.bcol[seg] + kx, b_row);
            }
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
      // Drain: the last S issued stages may still have loads in flight.  A
      // pair's loads complete on the even CTA's full barriers, which that CTA
      // drains; the odd CTA waits until the MMAs released its last stages
      // (a stage is released only after both CTAs' bytes for it landed), and
      // it leaves the kernel only after the closing cluster barrier, which
      // the even CTA reaches after its own drain.
      for (int i = 0; i < S; ++i) {
        if (--stage < 0) {
          stage = S - 1;
          phase ^= 1u;
        }
        if (CG == 1 || leader)
          tc::mbar_wait(tc::smem_u32(&full[stage]), phase, nullptr, kWaitBudget / 8);
        else
          tc::mbar_wait(tc::smem_u32(&empty[stage]), phase, nullptr, kWaitBudget / 8);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = unit; tile < total_tiles && ok; tile += n_units, ++it) {
        int g, m, n;
        decode(tile, g, m, n);
        const int n_valid = min(BN, grp_cnt[g] - n * BN);
        const uint32_t n_mma = (uint32_t)mma_width(n_valid);
        const uint32_t idesc = F8 ? tc::idesc_e4m3_f32(CG * kBM, n_mma)
                                  : tc::idesc_bf16_f32(CG * kBM, n_mma);
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
          for (int k = 0; k < 4; ++k) {  // 4 instructions of 32 bytes of K
            const uint64_t ad = tc::smem_desc_sw128(sa + k * 32);
            const uint64_t bd = tc::smem_desc_sw128(sb + k * 32);
            const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
            if (F8) {
              if (CG == 2) tc::mma_e4m3_pair(d_tmem, ad, bd, idesc, acc);
              else tc::mma_e4m3(d_tmem, ad, bd, idesc, acc);
            } else {
              if (CG == 2) tc::mma_bf16_pair(d_tmem, ad, bd, idesc, acc);
              else tc::mma_bf16(d_tmem, ad, bd, idesc, acc);
            }
          }
          if (CG == 2)
            tc::mma_commit_pair(tc::smem_u32(&empty[stage]), 0x3);
          else
            tc::mma_commit(tc::smem_u32(&empty[stage]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (CG == 2)
          tc::mma_commit_pair(tc::smem_u32(&tfull[b]), 0x3);
        else
          tc::mma_commit(tc::smem_u32(&tfull[b]));
      }
      if (!ok) {
        record_error(p.status, MOE_ERR_TIMEOUT);
        *abort_flag = 1;
        // Let every MMA issued so far finish before TMEM is released.
        if (CG == 2)
          tc::mma_commit_pair(tc::smem_u32(drain), 0x1);
        else
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
    for (int tile = unit; tile < total_tiles; tile += n_units, ++it) {
      int g, m, n;
      decode(tile, g, m, n);
      const int n_valid = min(BN, grp_cnt[g] - n * BN);
      const int tok0 = grp_beg[g] + n * BN;
      const int b = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      // the tile's token-row factors, fetched while the accumulator is being
      // computed, once every epilogue warp is done with the previous tile's
      if (p.b_scale) {
        named_sync_epi();
        for (int i = row; i < BN; i += 128) fac[i] = i < n_valid ? p.b_scale[tok0 + i] : 1.0f;
      }
      // The four epilogue warps share named barriers, so they take the
      // give-up decision together (the barrier also publishes fac).
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
      // E4M3: this thread's weight-row scale (gate/up: its TMEM row is a
      // gate row in lanes 0-63, an up row in lanes 64-127)
      float w_scale = 1.0f;
      if (F8) {
        if (p.mode == MODE_GATEUP) {
          const int hid = g * p.a_rows_per_group + (m * CG + (int)rank) * 64 + (row & 63);
          w_scale = p.a_scale[row >> 6][hid];
        } else {
          w_scale = p.a_scale[0][g * p.a_rows_per_group + (m * CG + (int)rank) * kBM + row];
        }
      }
      for (int c = 0; c < n_valid; c += 32) {
        float v[32];
        tc::tmem_ld_32x32b_x32(t_row + (uint32_t)c, v);
        if (F8 || p.b_scale) {  // row scales of A (E4M3) and of B (E4M3, or combine weights)
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = v[j] * w_scale * (p.b_scale ? fac[c + j] : 1.0f);
        }
        if (p.mode == MODE_GATEUP) {
#pragma unroll
          for (int j = 0; j < 32; ++j) epi[row * kEpiLd + j] = v[j];
          named_sync_epi();
          const int tok = c + lane;
          if (tok < n_valid) {
            float hv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              hv[i] = gated_act<ACT>(epi[(q * 16 + i) * kEpiLd + lane],
                                     epi[(64 + q * 16 + i) * kEpiLd + lane], p.beta_g, p.beta_u);
            const size_t o_el = (size_t)(tok0 + tok) * p.out_ld + g * p.out_col_group +
                                (m * CG + (int)rank) * 64 + q * 16;
            if (F8) {  // H as E4M3 codes, no scale
              uint32_t packed[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) packed[i] = e4m3x4_rn(&hv[4 * i]);
              *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + o_el) =
                  make_uint4(packed[0], packed[1], packed[2], packed[3]);
            } else {
              uint32_t packed[8];
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(hv[i], hv[i + 1]);
                packed[i >> 1] = *reinterpret_cast<uint32_t*>(&b2);
              }
              uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_el);
              o[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
              o[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
          }
          named_sync_epi();
        } else {
          const int col = g * p.out_col_group + (m * CG + (int)rank) * kBM + row;
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
      if (CG == 2) {
        // this CTA's 128 lanes are read: one arrival on the even CTA's barrier
        named_sync_epi();
        if (threadIdx.x == 64) tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(&tempty[b]), 0u));
      } else {
        tc::mbar_arrive(tc::smem_u32(&tempty[b]));
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  // A pair frees TMEM only when neither CTA's roles will touch the other
  // (remote arrivals, MMAs writing both CTAs' TMEM) any more.
  if (CG == 2) tc::cluster_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    if (CG == 2)
      tc::tmem_dealloc_pair(tmem_base, 2 * BN);
    else
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
// u8 = true: a matrix of E4M3 codes viewed as bytes, box 128 x box_rows (the
// same 128-byte rows and swizzle).
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
               bool u8 = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (u8 ? 1 : 2)};
  cuuint32_t box[2] = {(cuuint32_t)(u8 ? 2 * kBK : kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two CTAs that can be resident at once for a pair kernel (a GPC
// with an odd number of free SMs leaves one SM out), looked up once per
// device: a persistent pair kernel launches exactly that many, never more,
// so that no cluster waits for another to finish.
template <typename Kernel>
int resident_pairs(Kernel kernel, size_t smem, int dev) {
  static std::atomic<int> cached[kMaxDevices];
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n) return n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (unsigned)sm_count());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 0;
  }
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int BN, int S, int ACT, int CG, bool F8>
int launch_tc(const TcParams& p, int64_t units_upper, cudaStream_t st) {
  using L = Layout<BN, S, CG>;
  auto kernel = tc_grouped_gemm<BN, S, ACT, CG, F8>;
  const size_t smem = L::bytes(p.G);
  static std::atomic<bool> configured[kMaxDevices];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!device_slot(dev)) return MOE_ERR_CUDA;
  if (needs_setup(configured, dev)) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::bytes(1024)) != cudaSuccess)
      return MOE_ERR_CUDA;
    mark_setup(configured, dev);
  }
  MOE_PREFER_SHARED((tc_grouped_gemm<BN, S, ACT, CG, F8>));
  if (units_upper <= 0) return MOE_OK;
  if (CG == 1) {
    int64_t grid = sm_count();
    if (units_upper < grid) grid = units_upper;
    launch_pdl(kernel, dim3((unsigned)grid), dim3(kThreads), smem, st, p);
    return launch_status();
  }
  int64_t pairs = resident_pairs(kernel, L::bytes(1024), dev);
  if (pairs <= 0) return MOE_ERR_CUDA;
  if (units_upper < pairs) pairs = units_upper;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, p);
  if (e != cudaSuccess) pdl_launch_error() = e;
  return launch_status();
}

// Token tile width: 128 columns when groups average under 192 rows (a
// 256-wide tile would be mostly padding) or when 256-wide tiles would not
// give every SM (every pair, for CTA pairs) two tiles; 256 otherwise.
int pick_bn(int m_tiles, int64_t max_rows, int G, int cg) {
  if (max_rows < 192LL * G) return 128;
  const int64_t up256 = (int64_t)m_tiles * ((max_rows + 255) / 256 + G);
  return up256 >= 2LL * sm_count() / cg ? 256 : 128;
}

template <bool F8>
int launch_tc_typed(const TcParams& p, int64_t upper, int bn, int cg, cudaStream_t st) {
  const bool situ = p.mode == MODE_GATEUP && p.act_kind == MOE_ACT_SITU_GLU;
  if (cg == 2) {
    if (bn == 256)
      return situ ? launch_tc<256, 6, MOE_ACT_SITU_GLU, 2, F8>(p, upper, st)
                  : launch_tc<256, 6, MOE_ACT_SWIGLU, 2, F8>(p, upper, st);
    return situ ? launch_tc<128, 8, MOE_ACT_SITU_GLU, 2, F8>(p, upper, st)
                : launch_tc<128, 8, MOE_ACT_SWIGLU, 2, F8>(p, upper, st);
  }
  if (bn == 256)
    return situ ? launch_tc<256, 4, MOE_ACT_SITU_GLU, 1, F8>(p, upper, st)
                : launch_tc<256, 4, MOE_ACT_SWIGLU, 1, F8>(p, upper, st);
  return situ ? launch_tc<128, 6, MOE_ACT_SITU_GLU, 1, F8>(p, upper, st)
              : launch_tc<128, 6, MOE_ACT_SWIGLU, 1, F8>(p, upper, st);
}

int launch_tc_bn(const TcParams& p, int64_t max_rows, int bn, int cg, bool f8, cudaStream_t st) {
  const int64_t upper = (int64_t)p.m_tiles * ((max_rows + bn - 1) / bn + p.G);
  return f8 ? launch_tc_typed<true>(p, upper, bn, cg, st)
            : launch_tc_typed<false>(p, upper, bn, cg, st);
}

}  // namespace

size_t ffn_tc_ws_bytes(const moe_shape& s, int32_t /*width*/) {
  return align_up((size_t)s.T * s.k * s.h * 2, 256);
}

int launch_ffn_tc(const moe_shape& s, int32_t width, const __nv_bfloat16* x_rows,
                  const int32_t* offsets, const __nv_bfloat16* w_gate, const __nv_bfloat16* w_up,
                  const __nv_bfloat16* w_down, const moe_act& act, void* y_rows, void* ws,
                  cudaStream_t st, const float* row_w) {
  const int64_t R = (int64_t)s.T * s.k;
  if (R == 0) return MOE_OK;
  if (ffn_fused_ok(width, s.h, s.N))  // small h: both GEMMs in one launch, H stays on chip
    return launch_ffn_fused(s.N, R, width, s.h, x_rows, offsets, w_gate, w_up, w_down, act,
                            y_rows, st, row_w);
  __nv_bfloat16* H = static_cast<__nv_bfloat16*>(ws);
  int rc = tc_gateup(offsets, (int)R, s.N, x_rows, R, width, w_gate, w_up, s.h, act, H, s.h, 0,
                     st);
  if (rc != MOE_OK) return rc;
  TcSeg seg{w_down, (int64_t)s.N * width, s.h, 0, H, R, s.h, 0};
  return tc_store(offsets, (int)R, s.N, width, &seg, 1, y_rows,
                  MODE_STORE_F32, width, st, nullptr, row_w);
}

// Gate/up GEMM with the fused activation: for group g and its rows of X,
// out[row][g * out_col_group + j] = act(X W_gate[g]^T, X W_up[g]^T)[j], bf16.
int tc_gateup(const int32_t* offsets, int T, int G, const void* X, int64_t x_rows, int K,
              const void* w_gate, const void* w_up, int hidden, const moe_act& act, void* out,
              int out_ld, int out_col_group, cudaStream_t st, const TcF8* f8) {
  if (f8 && K % (2 * kBK) != 0) return MOE_ERR_UNSUPPORTED;
  TcParams p{};
  const int64_t rows_w = (int64_t)G * hidden;
  const int64_t max_rows = offsets ? x_rows : (int64_t)T * G;
  // CTA pairs take 128 hidden units (64 per CTA) per tile
  const int cg = hidden % 128 == 0 ? 2 : 1;
  const int m_tiles = hidden / (64 * cg);
  const int bn = pick_bn(m_tiles, max_rows, G, cg);
  const bool u8 = f8 != nullptr;
  if (!make_tmap(&p.maps[0], w_gate, rows_w, K, 64, u8) ||
      !make_tmap(&p.maps[1], w_up, rows_w, K, 64, u8) ||
      !make_tmap(&p.maps[2], X, x_rows, K, bn / cg, u8))
    return MOE_ERR_CUDA;
  if (f8) {
    p.a_scale[0] = f8->a_scale[0];
    p.a_scale[1] = f8->a_scale[1];
    p.b_scale = f8->b_scale;
  }
  p.maps[3] = p.maps[2];
  p.offsets = offsets;
  p.T = T;
  p.G = G;
  p.nseg = 1;
  p.seg_end[0] = K / (u8 ? 2 * kBK : kBK);
  p.a_rows_per_group = hidden;
  p.m_tiles = m_tiles;
  p.mode = MODE_GATEUP;
  p.act_kind = act.kind;
  p.beta_g = act.beta_gate;
  p.beta_u = act.beta_up;
  p.out = out;
  p.out_ld = out_ld;
  p.out_col_group = out_col_group;
  p.status = status_word();
  return launch_tc_bn(p, max_rows, bn, cg, u8, st);
}

// Plain GEMM over 1..3 K-segments accumulated into one output:
// out[row][g * m_rows + m] = sum_s (A_s[g * a_rows_s + arow_s + m] . B_s[row][bcol_s + ...]).
int tc_store(const int32_t* offsets, int T, int G, int m_rows, const TcSeg* segs, int nseg,
             void* out, int mode, int out_ld, cudaStream_t st, const TcF8* f8,
             const float* b_row_scale) {
  if (nseg < 1 || nseg > kMaxSeg) return MOE_ERR_INVALID_ARG;
  if (f8 && (nseg != 1 || segs[0].K % (2 * kBK) != 0)) return MOE_ERR_UNSUPPORTED;
  const bool u8 = f8 != nullptr;
  const int ke = u8 ? 2 * kBK : kBK;
  TcParams p{};
  const int64_t max_rows = offsets ? segs[0].b_rows : (int64_t)T * G;
  // CTA pairs take 256 output rows (128 per CTA) per tile
  const int cg = m_rows % (2 * kBM) == 0 ? 2 : 1;
  const int m_tiles = m_rows / (kBM * cg);
  const int bn = pick_bn(m_tiles, max_rows, G, cg);
  // distinct (pointer, rows, cols, box) tensor maps, at most four
  const void* key_p[4];
  int64_t key_r[4];
  int key_c[4], key_box[4];
  int nmaps = 0;
  auto map_of = [&](const void* ptr, int64_t rows, int cols, int box) -> int {
    for (int i = 0; i < nmaps; ++i)
      if (key_p[i] == ptr && key_r[i] == rows && key_c[i] == cols && key_box[i] == box) return i;
    if (nmaps >= 4) return -1;
    if (!make_tmap(&p.maps[nmaps], ptr, rows, cols, box, u8)) return -2;
    key_p[nmaps] = ptr;
    key_r[nmaps] = rows;
    key_c[nmaps] = cols;
    key_box[nmaps] = box;
    return nmaps++;
  };
  int kb = 0;
  for (int i = 0; i < nseg; ++i) {
    const int ia = map_of(segs[i].a, segs[i].a_rows, segs[i].K, kBM);
    const int ib = map_of(segs[i].b, segs[i].b_rows, segs[i].b_cols, bn / cg);
    if (ia == -1 || ib == -1) return MOE_ERR_UNSUPPORTED;
    if (ia < 0 || ib < 0) return MOE_ERR_CUDA;
    p.amap[i] = ia;
    p.bmap[i] = ib;
    kb += segs[i].K / ke;
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
  p.m_tiles = m_tiles;
  p.mode = mode;
  p.out = out;
  p.out_ld = out_ld;
  p.out_col_group = 0;
  p.status = status_word();
  p.b_scale = b_row_scale;
  if (f8) {
    p.a_scale[0] = f8->a_scale[0];
    p.b_scale = f8->b_scale;
  }
  return launch_tc_bn(p, max_rows, bn, cg, u8, st);
}

}  // namespace moe
