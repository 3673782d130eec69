// Token permutation: group the T*k dispatches by expert with a per-expert
// capacity (tutorial "Mixture of Experts MoE: how sparse activation saves
// compute", §3.5 capacity C, §3.6 grouping into per-expert [L_i, d] rows,
// §3.8 overflow and empty slots).
//
// Three launches, all deterministic (atomics only count, ranks come from
// scans):
//   1. permute_hist:    block b counts the experts of dispatches
//                       [256 b, 256 b + 256) -> hist[b][e]
//   2. permute_scan:    one block; per expert an exclusive scan over blocks
//                       (hist becomes the base rank of block b), L_e, the
//                       kept counts, their exclusive scan -> offsets, overflow
//                       and the totals
//   3. permute_scatter: block b ranks its dispatches stably (warp match +
//                       per-warp counts), keeps rank < C, writes row_of and
//                       perm_tok
#include "common.cuh"

namespace moe {
namespace {

constexpr int kChunk = 256;  // dispatches per block = 8 warps x 32 lanes

__global__ void __launch_bounds__(kChunk)
    permute_hist(const int32_t* __restrict__ idx, int64_t total, int N, int32_t* __restrict__ hist,
                 int* status) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ int32_t cnt[];
  for (int i = threadIdx.x; i < N; i += kChunk) cnt[i] = 0;
  __syncthreads();
  const int64_t x = (int64_t)blockIdx.x * kChunk + threadIdx.x;
  if (x < total) {
    const int e = idx[x];
    if (e >= 0 && e < N) {
      atomicAdd(&cnt[e], 1);
    } else {
      record_error(status, MOE_ERR_BOUNDS);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < N; i += kChunk) hist[(size_t)blockIdx.x * N + i] = cnt[i];
}

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ int block_exclusive_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_sums[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int before = w > 0 ? warp_sums[w - 1] : 0;
  if (total) *total = warp_sums[((blockDim.x + 31) >> 5) - 1];
  __syncthreads();
  return before + incl - v;
}

__device__ int block_sum(int v) {
  int t;
  block_exclusive_scan(v, &t);
  return t;
}

__global__ void __launch_bounds__(1024)
    permute_scan(int32_t* __restrict__ hist, int nblk, int N, int C, int32_t* __restrict__ counts,
                 int32_t* __restrict__ offsets, int32_t* __restrict__ overflow,
                 int32_t* __restrict__ totals) {
  pdl_wait();
  pdl_allow_next();
  const int e = threadIdx.x;
  int L = 0;
  if (e < N) {
    // eight loads in flight per round (the loop rewrites what it reads, so
    // the compiler would otherwise wait on each load)
    for (int b0 = 0; b0 < nblk; b0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = b0 + j < nblk ? hist[(size_t)(b0 + j) * N + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (b0 + j < nblk) hist[(size_t)(b0 + j) * N + e] = L;
        L += v[j];
      }
    }
  }
  const int kept = e < N ? ((C > 0 && L > C) ? C : L) : 0;
  const int of = (e < N && C > 0 && L > C) ? L - C : 0;
  const int empty = (e < N && C > 0 && L < C) ? C - L : 0;
  int kept_total = 0;
  const int off = block_exclusive_scan(kept, &kept_total);
  const int of_total = block_sum(of);
  const int empty_total = block_sum(empty);
  if (e < N) {
    counts[e] = L;
    offsets[e] = off;
    overflow[e] = of;
  }
  if (e == 0) {
    offsets[N] = kept_total;
    totals[0] = kept_total;
    totals[1] = of_total;
    totals[2] = empty_total;
  }
}

__global__ void __launch_bounds__(kChunk)
    permute_scatter(const int32_t* __restrict__ idx, int64_t total, int k, int N, int C,
                    const int32_t* __restrict__ base, const int32_t* __restrict__ offsets,
                    int32_t* __restrict__ perm_tok, int32_t* __restrict__ row_of,
                    const float* __restrict__ top_w, float* __restrict__ row_w) {
  pdl_wait();
  pdl_allow_next();
  extern __shared__ int32_t wcnt[];  // [8][N]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 8 * N; i += kChunk) wcnt[i] = 0;
  const int64_t x = (int64_t)blockIdx.x * kChunk + threadIdx.x;
  int e = -1;
  if (x < total) {
    e = idx[x];
    if (e < 0 || e >= N) e = -1;  // counted as an error by permute_hist
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int in_warp = __popc(peers & ((1u << lane) - 1u));
  __syncthreads();
  if (e >= 0 && in_warp == 0) wcnt[w * N + e] = __popc(peers);
  __syncthreads();
  if (x >= total) return;
  if (e < 0) {
    row_of[x] = -1;
    return;
  }
  int cross = 0;
  for (int v = 0; v < w; ++v) cross += wcnt[v * N + e];
  const int rank = base[(size_t)blockIdx.x * N + e] + cross + in_warp;
  if (C > 0 && rank >= C) {
    row_of[x] = -1;
  } else {
    const int r = offsets[e] + rank;
    row_of[x] = r;
    perm_tok[r] = (int32_t)(x / k);
    if (row_w) row_w[r] = top_w[x];  // the combine weight of grouped row r
  }
}

// Permutation in one launch for few experts (N <= 16), from the per-block
// expert counts the fused router wrote (router block r owns tokens
// [tpb r, tpb (r+1)), i.e. dispatches [tpb k r, tpb k (r+1))).  Block b of
// this kernel owns the dispatches of router blocks [R b, R (b+1)) (one thread
// each; R tpb k is a multiple of 32 near 256).  It loads all the
// counts into shared memory at once, sums those of the blocks before it (its
// base ranks) and of all blocks (L_e, offsets), ranks its dispatches stably
// as permute_scatter does and writes row_of / perm_tok.
constexpr int kDispatchMaxHist = 8192;  // nblk * N ints held in shared memory

__global__ void __launch_bounds__(512)
    dispatch_small(const int32_t* __restrict__ idx, int64_t total, int k, int N, int C,
                   const int32_t* __restrict__ hist, int nblk, int rblk_per_block,
                   int32_t* __restrict__ counts,
                   int32_t* __restrict__ offsets, int32_t* __restrict__ overflow,
                   int32_t* __restrict__ totals, int32_t* __restrict__ perm_tok,
                   int32_t* __restrict__ row_of, const float* __restrict__ top_w,
                   float* __restrict__ row_w, int* status) {
  pdl_wait();
  pdl_allow_next();
  __shared__ int hist_s[kDispatchMaxHist];
  __shared__ int base_s[16], L_s[16], off_s[17];
  __shared__ int wcnt[16][16];
  const int b = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nh = nblk * N;
  for (int i0 = threadIdx.x; i0 < nh; i0 += 8 * blockDim.x) {
    int v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + j * blockDim.x;
      v[j] = i < nh ? hist[i] : 0;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + j * blockDim.x;
      if (i < nh) hist_s[i] = v[j];
    }
  }
  for (int i = threadIdx.x; i < 16 * 16; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  if (threadIdx.x < N) {
    const int e = threadIdx.x;
    const int first = b * rblk_per_block;  // first router block of this block's dispatches
    int base = 0, tot = 0;
    for (int i = 0; i < nblk; ++i) {
      const int v = hist_s[i * N + e];
      base += i < first ? v : 0;
      tot += v;
    }
    base_s[e] = base;
    L_s[e] = tot;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0, of = 0, empty = 0;
    for (int e = 0; e < N; ++e) {
      const int L = L_s[e];
      off_s[e] = run;
      run += (C > 0 && L > C) ? C : L;
      if (C > 0 && L > C) of += L - C;
      if (C > 0 && L < C) empty += C - L;
    }
    off_s[N] = run;
    if (b == 0) {
      for (int e = 0; e < N; ++e) {
        counts[e] = L_s[e];
        offsets[e] = off_s[e];
        overflow[e] = (C > 0 && L_s[e] > C) ? L_s[e] - C : 0;
      }
      offsets[N] = run;
      totals[0] = run;
      totals[1] = of;
      totals[2] = empty;
    }
  }
  const int64_t x = (int64_t)b * blockDim.x + threadIdx.x;
  int e = -1;
  if (x < total) {
    e = idx[x];
    if (e < 0 || e >= N) {
      record_error(status, MOE_ERR_BOUNDS);
      e = -1;
    }
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int in_warp = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && in_warp == 0) wcnt[w][e] = __popc(peers);
  __syncthreads();
  if (x >= total) return;
  int row = -1;
  if (e >= 0) {
    int cross = 0;
    for (int v = 0; v < w; ++v) cross += wcnt[v][e];
    const int rank = base_s[e] + cross + in_warp;
    if (!(C > 0 && rank >= C)) {
      row = off_s[e] + rank;
      perm_tok[row] = (int32_t)(x / k);
      if (row_w) row_w[row] = top_w[x];
    }
  }
  row_of[x] = row;
}

}  // namespace

size_t permute_ws_bytes(const moe_shape& s) {
  const int64_t total = (int64_t)s.T * s.k;
  const int64_t nblk = (total + kChunk - 1) / kChunk;
  return align_up((size_t)(nblk > 0 ? nblk : 1) * s.N * 4, 256);
}

int launch_permute(const moe_shape& s, const int32_t* top_idx, int32_t* counts, int32_t* offsets,
                   int32_t* perm_tok, int32_t* row_of, int32_t* overflow, int32_t* totals,
                   void* ws, cudaStream_t st, const float* top_w, float* row_w) {
  const int64_t total = (int64_t)s.T * s.k;
  const int nblk = (int)((total + kChunk - 1) / kChunk);
  int32_t* hist = static_cast<int32_t*>(ws);
  if (nblk > 0) {
    MOE_PREFER_SHARED((permute_hist));
    launch_pdl(permute_hist, dim3(nblk), dim3(kChunk), (size_t)s.N * 4, st, top_idx, total, s.N, hist, status_word());
  }
  MOE_PREFER_SHARED((permute_scan));
  launch_pdl(permute_scan, dim3(1), dim3(1024), 0, st, hist, nblk, s.N, s.capacity, counts, offsets, overflow, totals);
  if (nblk > 0) {
    MOE_PREFER_SHARED((permute_scatter));
    launch_pdl(permute_scatter, dim3(nblk), dim3(kChunk), (size_t)s.N * 8 * 4, st, top_idx,
               total, s.k, s.N, s.capacity, hist, offsets, perm_tok, row_of, top_w, row_w);
  }
  return launch_status();
}

bool dispatch_small_ok(const moe_shape& s) {
  const int tpb = route_tokens_per_block(s.N);
  const int64_t nblk = (s.T + tpb - 1) / tpb;
  return s.N <= 16 && s.k <= 16 && nblk * s.N <= kDispatchMaxHist;
}

int launch_dispatch_small(const moe_shape& s, const int32_t* top_idx, const int32_t* hist,
                          int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                          int32_t* overflow, int32_t* totals, cudaStream_t st,
                          const float* top_w, float* row_w) {
  const int tpb = route_tokens_per_block(s.N);
  const int nblk = (s.T + tpb - 1) / tpb;
  const int per = tpb * s.k;  // dispatches of one router block
  int g = per, h = 32;        // lcm(per, 32)
  while (h) {
    const int t = g % h;
    g = h;
    h = t;
  }
  const int L = per / g * 32;
  const int threads = L * (L < 256 ? 256 / L : 1);
  const int rpb = threads / per;
  const int64_t total = (int64_t)s.T * s.k;
  const int blocks = (int)((total + threads - 1) / threads);
  MOE_PREFER_SHARED((dispatch_small));
  launch_pdl(dispatch_small, dim3(blocks > 0 ? blocks : 1), dim3(threads), 0, st, top_idx, total,
             s.k, s.N, s.capacity, hist, nblk, rpb, counts, offsets, overflow, totals, perm_tok,
             row_of, top_w, row_w, status_word());
  return launch_status();
}

}  // namespace moe

extern "C" size_t moe_permute_workspace_bytes(const moe_shape* shape) {
  if (!moe::shape_ok(shape)) return 0;
  return moe::permute_ws_bytes(*shape);
}

extern "C" int moe_permute(const moe_shape* shape, const int32_t* top_idx, int32_t* counts,
                           int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                           int32_t* overflow, int32_t* totals, void* ws, size_t ws_bytes,
                           void* stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_INVALID_ARG;
  if (!counts || !offsets || !overflow || !totals) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!top_idx || !perm_tok || !row_of)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < permute_ws_bytes(*shape)) return MOE_ERR_WORKSPACE;
  return launch_permute(*shape, top_idx, counts, offsets, perm_tok, row_of, overflow, totals, ws,
                        as_stream(stream));
}

// ------------------------------------------------- allocation-free variant
// Some callers cannot allocate device memory when they call in: a C program
// that loads only this library and owns no device allocator, or a host
// framework whose memory planner hands out every device byte in advance and
// forbids allocation at call time.  moe_permute_noalloc serves them with the
// same kernels as moe_permute, taking its block-count scratch from this fixed
// array instead of a caller workspace.  Every GPU that loads the library
// holds the array until the process exits.
static __device__ __align__(256) int32_t g_permute_noalloc_scratch[262144];  // 1 MiB

namespace moe {
namespace {

// Device address of the scratch array for the current device, looked up once
// per device with that device current (in host code the array's name is only a
// host-side stand-in and must not be handed to a kernel).
int32_t* noalloc_scratch() {
  static std::atomic<int32_t*> addr[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || !device_slot(dev)) return nullptr;
  int32_t* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_noalloc_scratch) != cudaSuccess) return nullptr;
    a = static_cast<int32_t*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace
}  // namespace moe

extern "C" int moe_permute_noalloc(const moe_shape* shape, const int32_t* top_idx,
                                   int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                                   int32_t* row_of, int32_t* overflow, int32_t* totals,
                                   void* stream) {
  using namespace moe;
  if (!shape_ok(shape)) return MOE_ERR_INVALID_ARG;
  if (!counts || !offsets || !overflow || !totals) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!top_idx || !perm_tok || !row_of)) return MOE_ERR_INVALID_ARG;
  if (permute_ws_bytes(*shape) > sizeof(g_permute_noalloc_scratch)) return MOE_ERR_WORKSPACE;
  int32_t* scratch = noalloc_scratch();
  if (!scratch) return MOE_ERR_CUDA;
  return launch_permute(*shape, top_idx, counts, offsets, perm_tok, row_of, overflow, totals,
                        scratch, as_stream(stream));
}
