// Expert parallelism, device side: the all-to-all dispatch and combine that
// the tutorial "Mixture of Experts MoE: how sparse activation saves compute"
// names as the multi-device cost of splitting the experts over devices, fused
// with the gather and with the weighted combine.
//
// R ranks, expert e on rank e / (N / R).  Each rank holds, in its own memory,
// a receive buffer of bf16 rows (with one combine weight per row), an output
// buffer of fp32 rows, R arrival flags and one done flag; every rank can
// address every rank's buffers (peer memory over NVLink, or one device).
// One step, with the exchange plan of moe_ep_plan (rows of one expert from
// rank 0 first, then rank 1, ..., each in token order, capacity in that
// order):
//   dispatch  (source)  each kept dispatch's token row and combine weight are
//                       stored straight into its owner's receive buffer at the
//                       plan's row (the gather and the all-to-all in one
//                       kernel); the last CTA raises arrive[rank] on every
//                       owner (release, system scope)
//   expert FFN (owner)  waits until every source has arrived, runs the
//                       grouped SwiGLU experts on its receive buffer and
//                       stores fp32 rows a * F(u) into its output buffer,
//                       then raises its done flag
//   combine   (source)  waits for every owner's done flag and forms
//                       y_t = sum over kept slots of the owners' output rows,
//                       read straight from their memory (the all-to-all back
//                       and the combine in one kernel)
// Flags carry the step number (epoch), so they are never reset.  Every wait
// is bounded (2 s of device time) and records MOE_ERR_TIMEOUT.  Loads from a
// peer are plain loads: no TMA, no multicast.
#include "common.cuh"
#include "grid_sync.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void st_release_sys(unsigned* p, unsigned v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_sys(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Epochs grow by one per step; "reached" tolerates wrap-around.
__device__ __forceinline__ bool reached(unsigned v, unsigned epoch) {
  return (int)(v - epoch) >= 0;
}

// One thread waits until every flag flags[i * stride] has reached epoch.
__device__ bool wait_flags(const unsigned* const* flags_of, const unsigned* flags, int n,
                           int stride, unsigned epoch, int* status) {
  const unsigned long long t0 = global_ns();
  for (int i = 0; i < n; ++i) {
    const unsigned* f = flags_of ? flags_of[i] : flags + (size_t)i * stride;
    unsigned polls = 0;
    while (!reached(ld_acquire_sys(f), epoch)) {
      if ((++polls & 63u) == 0 && global_ns() - t0 > kBarrierBudgetNs) {
        record_error(status, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

__global__ void ep_wait_arrivals(const unsigned* arrive, int world, unsigned epoch, int* status,
                                 int* go) {
  pdl_wait();
  if (threadIdx.x == 0) *go = wait_flags(nullptr, arrive, world, 1, epoch, status) ? 1 : 0;
  pdl_allow_next();
}

__global__ void ep_signal(unsigned* flag, unsigned epoch) {
  pdl_wait();
  if (threadIdx.x == 0) {
    __threadfence_system();
    st_release_sys(flag, epoch);
  }
}

struct DispatchParams {
  const uint4* u;            // [T][d] bf16, as 16-byte vectors
  int vec;                   // 16-byte vectors per row
  int T, k, N, E, world, rank;
  const int32_t* perm_tok;   // local capacity-0 permutation
  const int32_t* offsets;    // [N+1]
  const int32_t* row_of;     // [T][k]
  const float* top_w;        // [T][k]
  const int32_t* kept;       // [N] plan: my kept dispatches per expert
  const int32_t* send_base;  // [N] plan: first row in the owner's receive buffer
  int recv_capacity;         // rows of every receive buffer
  uint4* const* recv_rows;   // [world] owners' receive buffers
  float* const* recv_w;      // [world] owners' row weights
  unsigned* const* arrive;   // [world] owners' arrival flag arrays [world]
  unsigned epoch;
  unsigned* blocks_done;     // local counter, zeroed before the launch
  int* status;
};

// One warp per local grouped row; the last CTA to finish raises the flags.
__global__ void __launch_bounds__(256) ep_dispatch(const __grid_constant__ DispatchParams p) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int rows = p.offsets[p.N];
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += (gridDim.x * blockDim.x) >> 5) {
    int lo = 0, hi = p.N;  // expert of row r: offsets[lo] <= r < offsets[lo + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.offsets[mid] <= r) lo = mid; else hi = mid;
    }
    const int e = lo, j = r - p.offsets[e];
    if (j >= p.kept[e]) continue;  // beyond this rank's share of the capacity
    const int t = p.perm_tok[r];
    if (t < 0 || t >= p.T) {
      if (lane == 0) record_error(p.status, MOE_ERR_BOUNDS);
      continue;
    }
    const int o = e / p.E, dst = p.send_base[e] + j;
    if (dst < 0 || dst >= p.recv_capacity) {  // a plan that does not fit the buffers
      if (lane == 0) record_error(p.status, MOE_ERR_BOUNDS);
      continue;
    }
    const uint4* src = p.u + (size_t)t * p.vec;
    uint4* out = p.recv_rows[o] + (size_t)dst * p.vec;
    for (int v = lane; v < p.vec; v += 32) out[v] = src[v];
    if (lane == 0) {
      float a = 0.0f;
      for (int s = 0; s < p.k; ++s)
        if (p.row_of[(size_t)t * p.k + s] == r) a = p.top_w[(size_t)t * p.k + s];
      p.recv_w[o][dst] = a;
    }
  }
  // every row this CTA stored is visible system-wide before the count
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(p.blocks_done, 1u);
    if (prev == gridDim.x - 1) {  // the last CTA: all rows of the step are out
      __threadfence_system();
      for (int o = 0; o < p.world; ++o) st_release_sys(p.arrive[o] + p.rank, p.epoch);
    }
  }
  pdl_allow_next();
}

struct CombineParams {
  int T, k, N, E, world, w4;  // w4: float4 vectors per row
  int recv_capacity;          // rows of every output buffer
  const int32_t* top_idx;
  const int32_t* row_of;     // local capacity-0 permutation
  const int32_t* offsets;
  const int32_t* kept;
  const int32_t* send_base;
  const float4* const* out_rows;  // [world] owners' weighted output rows (fp32)
  const unsigned* const* done;   // [world] owners' done flags
  unsigned epoch;
  __nv_bfloat16* y;
  int* status;
};

// One warp per token: wait (one thread per CTA) for every owner's done flag,
// then y_t = sum over kept slots (ascending s) of the owner's row, fp32 sum.
__global__ void __launch_bounds__(256) ep_combine(const __grid_constant__ CombineParams p) {
  pdl_wait();
  __shared__ int ok;
  if (threadIdx.x == 0) ok = wait_flags(p.done, nullptr, p.world, 0, p.epoch, p.status) ? 1 : 0;
  __syncthreads();
  if (!ok) return;
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < p.T;
       t += (gridDim.x * blockDim.x) >> 5) {
    for (int c = lane; c < p.w4; c += 32) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; s < p.k; ++s) {
        const int r = p.row_of[(size_t)t * p.k + s];
        const int e = p.top_idx[(size_t)t * p.k + s];
        if (r < 0 || e < 0 || e >= p.N) continue;
        const int j = r - p.offsets[e];
        if (j < 0 || j >= p.kept[e]) continue;  // dropped by the capacity
        const int row = p.send_base[e] + j;
        if (row < 0 || row >= p.recv_capacity) {  // a plan that does not fit the buffers
          record_error(p.status, MOE_ERR_BOUNDS);
          continue;
        }
        const float4 v = p.out_rows[e / p.E][(size_t)row * p.w4 + c];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 o;
      o.x = *reinterpret_cast<uint32_t*>(&lo);
      o.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(p.y + (size_t)t * p.w4 * 4)[c] = o;
    }
  }
  pdl_allow_next();
}

int warps_grid(int64_t warps) {
  int64_t b = (warps + 7) / 8;
  if (b > 148 * 8) b = 148 * 8;
  return (int)(b > 0 ? b : 1);
}

bool buffers_ok(const moe_ep_buffers* b, const moe_shape* s) {
  if (!b || !shape_ok(s)) return false;
  if (b->world < 1 || b->rank < 0 || b->rank >= b->world || s->N % b->world != 0) return false;
  if (b->recv_capacity < 0 || s->d % 8 != 0) return false;
  return b->recv_rows && b->recv_w && b->out_rows && b->arrive && b->done &&
         b->peer_recv_rows && b->peer_recv_w && b->peer_out_rows && b->peer_arrive &&
         b->peer_done && aligned16(b->recv_rows) && aligned16(b->out_rows);
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_ep_workspace_bytes(const moe_shape* expert_shape) {
  // the dispatch's CTA counter (256 bytes) and, for the owner's experts, the
  // expert FFN's workspace (expert_shape: T = receive capacity, k = 1,
  // N = experts per rank)
  if (!moe::shape_ok(expert_shape)) return 0;
  return 256 + moe::ffn_tc_ws_bytes(*expert_shape, expert_shape->d);
}

extern "C" int moe_ep_dispatch(const moe_shape* shape, const moe_ep_buffers* bufs, uint32_t epoch,
                               const void* u, const int32_t* perm_tok, const int32_t* offsets,
                               const int32_t* row_of, const float* top_w, const int32_t* kept,
                               const int32_t* send_base, void* ws, size_t ws_bytes,
                               void* stream) {
  using namespace moe;
  if (!buffers_ok(bufs, shape)) return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (!offsets || !kept || !send_base || (s.T > 0 && (!u || !perm_tok || !row_of || !top_w)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(u)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  DispatchParams p{};
  p.u = static_cast<const uint4*>(u);
  p.vec = s.d / 8;
  p.T = s.T;
  p.k = s.k;
  p.N = s.N;
  p.E = s.N / bufs->world;
  p.world = bufs->world;
  p.rank = bufs->rank;
  p.perm_tok = perm_tok;
  p.offsets = offsets;
  p.row_of = row_of;
  p.top_w = top_w;
  p.kept = kept;
  p.send_base = send_base;
  p.recv_capacity = bufs->recv_capacity;
  p.recv_rows = reinterpret_cast<uint4* const*>(bufs->peer_recv_rows);
  p.recv_w = bufs->peer_recv_w;
  p.arrive = bufs->peer_arrive;
  p.epoch = epoch;
  p.blocks_done = static_cast<unsigned*>(ws);
  p.status = status_word();
  if (cudaMemsetAsync(ws, 0, sizeof(unsigned), st) != cudaSuccess) return MOE_ERR_CUDA;
  MOE_PREFER_SHARED((ep_dispatch));
  // at least one CTA, so the arrival flags are raised even with no rows
  launch_pdl(ep_dispatch, dim3(warps_grid((int64_t)s.T * s.k)), dim3(256), 0, st, p);
  return launch_status();
}

extern "C" int moe_ep_expert_ffn(const moe_shape* expert_shape, const moe_ep_buffers* bufs,
                                 uint32_t epoch, const int32_t* recv_offsets, const void* w_gate,
                                 const void* w_up, const void* w_down, const moe_act* act,
                                 void* ws, size_t ws_bytes, void* stream) {
  using namespace moe;
  if (!shape_ok(expert_shape) || !bufs || !act || !recv_offsets || !w_gate || !w_up || !w_down)
    return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *expert_shape;  // T = receive capacity, k = 1, N = local experts
  if (s.k != 1 || s.T != bufs->recv_capacity || s.h % 64 != 0 || s.d % 128 != 0)
    return MOE_ERR_INVALID_ARG;
  if (bufs->world < 1 || bufs->rank < 0 || bufs->rank >= bufs->world || !bufs->recv_rows ||
      !bufs->recv_w || !bufs->out_rows || !bufs->arrive || !bufs->done)
    return MOE_ERR_INVALID_ARG;
  if (act->kind != MOE_ACT_SWIGLU &&
      !(act->kind == MOE_ACT_SITU_GLU && act->beta_gate > 0.0f && act->beta_up > 0.0f))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(bufs->recv_rows) || !aligned16(bufs->out_rows))
    return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < 256 + ffn_tc_ws_bytes(s, s.d)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  int* go = static_cast<int*>(ws);
  MOE_PREFER_SHARED((ep_wait_arrivals));
  launch_pdl(ep_wait_arrivals, dim3(1), dim3(32), 0, st, (const unsigned*)bufs->arrive,
             bufs->world, epoch, status_word(), go);
  int rc = launch_status();
  if (rc != MOE_OK) return rc;
  rc = launch_ffn_tc(s, s.d, static_cast<const __nv_bfloat16*>(bufs->recv_rows), recv_offsets,
                     static_cast<const __nv_bfloat16*>(w_gate),
                     static_cast<const __nv_bfloat16*>(w_up),
                     static_cast<const __nv_bfloat16*>(w_down), *act, bufs->out_rows,
                     static_cast<char*>(ws) + 256, st, bufs->recv_w);
  if (rc != MOE_OK) return rc;
  MOE_PREFER_SHARED((ep_signal));
  launch_pdl(ep_signal, dim3(1), dim3(32), 0, st, (unsigned*)bufs->done, epoch);
  return launch_status();
}

extern "C" int moe_ep_combine(const moe_shape* shape, const moe_ep_buffers* bufs, uint32_t epoch,
                              const int32_t* top_idx, const int32_t* row_of,
                              const int32_t* offsets, const int32_t* kept,
                              const int32_t* send_base, void* y, void* stream) {
  using namespace moe;
  if (!buffers_ok(bufs, shape)) return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (!offsets || !kept || !send_base || (s.T > 0 && (!top_idx || !row_of || !y)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  CombineParams p{};
  p.T = s.T;
  p.k = s.k;
  p.N = s.N;
  p.E = s.N / bufs->world;
  p.world = bufs->world;
  p.w4 = s.d / 4;
  p.recv_capacity = bufs->recv_capacity;
  p.top_idx = top_idx;
  p.row_of = row_of;
  p.offsets = offsets;
  p.kept = kept;
  p.send_base = send_base;
  p.out_rows = reinterpret_cast<const float4* const*>(bufs->peer_out_rows);
  p.done = reinterpret_cast<const unsigned* const*>(bufs->peer_done);
  p.epoch = epoch;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.status = status_word();
  MOE_PREFER_SHARED((ep_combine));
  launch_pdl(ep_combine, dim3(warps_grid(s.T)), dim3(256), 0, as_stream(stream), p);
  return launch_status();
}
