// The layer backward: gradients of L = sum_t dy_t . y_t (+ alpha N sum f_i P_i)
// for the layer of the tutorial "Mixture of Experts MoE: how sparse
// activation saves compute" (§3.1 expert F, §3.2 router and combine, §3.4
// P_i, §3.7 the balancing term's gradient with f held fixed), with the
// selected sets and the capacity drops of the forward held fixed (top-k and
// the capacity cut are piecewise constant); only the selected experts of
// kept dispatches receive gradient, the property the Stable LatentMoE demo
// document tests.
//
// Per step (bf16 experts, fp32 gradients), all on the caller's stream:
//   pad_offsets  each expert's kept rows start at a multiple of 64 (zero rows
//                between), so the weight-gradient GEMMs' K-blocks stay inside
//                one expert
//   gather       x rows, dy rows, a * dy rows and a per padded row
//   G, V         the forward's pre-activations recomputed (two tcgen05 GEMMs)
//   H            SiLU(g') v' as bf16 (elementwise)
//   dgrad_act    dH' = dy W_down (tcgen05, W_down read MN-major); epilogue:
//                dG, dV and the partial sums of dH' . H (da = dy . F)
//   dgrad_x      dX = dG W_gate + dV W_up (tcgen05, weights read MN-major)
//   wgrad        dW_gate = dG^T X, dW_up = dV^T X, dW_down = (a dy)^T H
//   dz           softmax / renormalisation backward plus the §3.7 term
//   du           du_t = sum over kept slots of dX rows + sum_j dz_tj W_route_j
//   dW_route     sum_t dz_t u_t^T
// Every sum is in a fixed order, so the gradients are reproducible bit for
// bit run to run.
#include <algorithm>

#include "bwd.cuh"

namespace moe {

namespace {

// One warp: pad[e] = sum over e' < e of round_up(offsets[e'+1] - offsets[e'], 64).
__global__ void pad_offsets(const int32_t* __restrict__ offsets, int N, int32_t* __restrict__ pad) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x;
  int carry = 0;
  for (int base = 0; base < N; base += 32) {
    const int e = base + lane;
    int c = 0;
    if (e < N) {
      c = offsets[e + 1] - offsets[e];
      c = c < 0 ? 0 : (c + 63) & ~63;
    }
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (e < N) pad[e] = carry + incl - c;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) pad[N] = carry;
}

struct GatherParams {
  const uint4* u;           // [T][d] bf16, nullable: x rows and a not written
  const uint4* dy;          // [T][d] bf16, nullable: dy rows not written
  int vec, T, k, N;
  const int32_t* offsets;   // [N+1] forward grouped layout
  const int32_t* pad;       // [N+1]
  const int32_t* perm_tok;  // [kept]
  const int32_t* row_of;    // [T][k]
  const float* top_w;       // [T][k]
  int max_rows;             // padded rows the buffers hold
  uint4* x;                 // [rows][d]
  uint4* dyr;               // [rows][d] dy of the row's token
  uint4* dyw;               // [rows][d] a * dy
  float* a;                 // [rows]
  int* status;
};

// One warp per padded row: the token's rows, or zeros in the padding.
__global__ void __launch_bounds__(256) bwd_gather(const __grid_constant__ GatherParams p) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  int rows = p.pad[p.N];
  if (rows > p.max_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(p.status, MOE_ERR_BOUNDS);
    rows = p.max_rows;
  }
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += (gridDim.x * blockDim.x) >> 5) {
    int lo = 0, hi = p.N;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.pad[mid] <= r) lo = mid; else hi = mid;
    }
    const int e = lo, j = r - p.pad[e];
    const int src = p.offsets[e] + j;
    int t = -1;
    float a = 0.0f;
    if (j < p.offsets[e + 1] - p.offsets[e]) {
      t = p.perm_tok[src];
      if (t < 0 || t >= p.T) {
        if (lane == 0) record_error(p.status, MOE_ERR_BOUNDS);
        t = -1;
      } else {
        for (int s = 0; s < p.k; ++s)
          if (p.row_of[(size_t)t * p.k + s] == src) a = p.top_w[(size_t)t * p.k + s];
      }
    }
    if (p.u) {
      uint4* xo = p.x + (size_t)r * p.vec;
      for (int v = lane; v < p.vec; v += 32)
        xo[v] = t < 0 ? make_uint4(0, 0, 0, 0) : p.u[(size_t)t * p.vec + v];
      if (lane == 0) p.a[r] = a;
    }
    if (p.dy) {
      uint4* d1 = p.dyr + (size_t)r * p.vec;
      uint4* d2 = p.dyw + (size_t)r * p.vec;
      for (int v = lane; v < p.vec; v += 32) {
        if (t < 0) {
          d1[v] = d2[v] = make_uint4(0, 0, 0, 0);
          continue;
        }
        const uint4 g = p.dy[(size_t)t * p.vec + v];
        d1[v] = g;
        float f[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(&g), f);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          __nv_bfloat162 b2 = __floats2bfloat162_rn(a * f[2 * i], a * f[2 * i + 1]);
          w[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        d2[v] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// H = bf16(act(g, v)) elementwise over [rows][h] (8 per thread).
template <int ACT>
__global__ void __launch_bounds__(256)
    bwd_hidden(const __nv_bfloat16* __restrict__ g, const __nv_bfloat16* __restrict__ v,
               int64_t n8, float bg, float bu, __nv_bfloat16* __restrict__ H) {
  pdl_wait();
  pdl_allow_next();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    float a[8], b[8];
    load8(g + i * 8, a);
    load8(v + i * 8, b);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float h0 = a[2 * j], v0 = b[2 * j], h1 = a[2 * j + 1], v1 = b[2 * j + 1];
      if (ACT == MOE_ACT_SITU_GLU) {
        h0 = bg * tanhf(h0 / bg);
        h1 = bg * tanhf(h1 / bg);
        v0 = bu * tanhf(v0 / bu);
        v1 = bu * tanhf(v1 / bu);
      }
      __nv_bfloat162 b2 = __floats2bfloat162_rn(silu(h0) * v0, silu(h1) * v1);
      w[j] = *reinterpret_cast<uint32_t*>(&b2);
    }
    reinterpret_cast<uint4*>(H)[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Padded row of dispatch (t, s), or -1 when the capacity dropped it.
__device__ __forceinline__ int padded_row(const int32_t* row_of, const int32_t* top_idx,
                                          const int32_t* offsets, const int32_t* pad, int N,
                                          size_t x) {
  const int r = row_of[x], e = top_idx[x];
  if (r < 0 || e < 0 || e >= N) return -1;
  return pad[e] + (r - offsets[e]);
}

struct DzParams {
  int T, N, k, renorm, m_tiles;
  const int32_t* top_idx;
  const float* top_w;
  const float* probs;     // [T][N]
  const int32_t* row_of;
  const int32_t* offsets;
  const int32_t* pad;
  const float* da_part;   // [rows][m_tiles]
  const float* f;         // nullable
  float alpha;
  float* dz;              // [T][N]
};

// One warp per token.  da_s = dy_t . F (the partial sums over the hidden
// tiles in order), then dp, the softmax backward and the balancing term.
__global__ void __launch_bounds__(256) bwd_dz(const __grid_constant__ DzParams p) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= p.T) return;
  const size_t x0 = (size_t)t * p.k;
  // slot sums of this token: lane s < k holds da_s, a_s and p_{e_s}
  float da = 0.0f, a = 0.0f, ps = 0.0f;
  int e = -1;
  if (lane < p.k) {
    e = p.top_idx[x0 + lane];
    a = p.top_w[x0 + lane];
    ps = (e >= 0 && e < p.N) ? p.probs[(size_t)t * p.N + e] : 0.0f;
    const int r = padded_row(p.row_of, p.top_idx, p.offsets, p.pad, p.N, x0 + lane);
    if (r >= 0)
      for (int m = 0; m < p.m_tiles; ++m) da += p.da_part[(size_t)r * p.m_tiles + m];
  }
  // renormalised: dp_{e_s} = (da_s - sum_r a_r da_r) / sum_r p_{e_r}; else dp = da
  float ssum = ps, ada = a * da;
  for (int o = 16; o >= 1; o >>= 1) {
    ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    ada += __shfl_xor_sync(0xffffffffu, ada, o);
  }
  const float dp = lane < p.k ? (p.renorm ? (da - ada) / ssum : da) : 0.0f;
  // sum_i p_i dp_i over the selected set
  float pdp = ps * dp;
  for (int o = 16; o >= 1; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
  float fbar = 0.0f;
  if (p.f) {
    for (int j = lane; j < p.N; j += 32) fbar += p.f[j] * p.probs[(size_t)t * p.N + j];
    for (int o = 16; o >= 1; o >>= 1) fbar += __shfl_xor_sync(0xffffffffu, fbar, o);
  }
  const float c = p.alpha * (float)p.N / (float)p.T;
  for (int j0 = 0; j0 < p.N; j0 += 32) {  // every lane takes part in the shuffles
    const int j = j0 + lane;
    float dpj = 0.0f;
    for (int s = 0; s < p.k; ++s) {
      const int es = __shfl_sync(0xffffffffu, e, s);
      const float dps = __shfl_sync(0xffffffffu, dp, s);
      if (es == j) dpj = dps;
    }
    if (j < p.N) {
      const float pj = p.probs[(size_t)t * p.N + j];
      float g = pj * (dpj - pdp);
      if (p.f) g += c * pj * (p.f[j] - fbar);
      p.dz[(size_t)t * p.N + j] = g;
    }
  }
}

struct DuParams {
  int T, N, k, d;
  const int32_t* top_idx;
  const int32_t* row_of;
  const int32_t* offsets;
  const int32_t* pad;
  const float* dX;        // [rows][d], nullable: no expert rows
  const float* dz;        // [T][N]
  const float* w_route;   // [N][d], nullable: no router term
  float* du;              // [T][d]
  int add;                // accumulate into du instead of overwriting it
};

// One warp per token: the kept slots' dX rows in slot order, then the router
// term in expert order.
__global__ void __launch_bounds__(256) bwd_du(const __grid_constant__ DuParams p) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < p.T;
       t += (gridDim.x * blockDim.x) >> 5) {
    const size_t x0 = (size_t)t * p.k;
    for (int c = lane * 4; c < p.d; c += 128) {
      float4 acc = p.add ? *reinterpret_cast<const float4*>(p.du + (size_t)t * p.d + c)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s = 0; p.dX && s < p.k; ++s) {
        const int r = padded_row(p.row_of, p.top_idx, p.offsets, p.pad, p.N, x0 + s);
        if (r < 0) continue;
        const float4 v = *reinterpret_cast<const float4*>(p.dX + (size_t)r * p.d + c);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      for (int j = 0; p.w_route && j < p.N; ++j) {
        const float z = p.dz[(size_t)t * p.N + j];
        const float4 w = *reinterpret_cast<const float4*>(p.w_route + (size_t)j * p.d + c);
        acc.x = fmaf(z, w.x, acc.x);
        acc.y = fmaf(z, w.y, acc.y);
        acc.z = fmaf(z, w.z, acc.z);
        acc.w = fmaf(z, w.w, acc.w);
      }
      *reinterpret_cast<float4*>(p.du + (size_t)t * p.d + c) = acc;
    }
  }
}

// dW_route[j][c] = sum_t dz[t][j] u[t][c]: one thread per (j, c), tokens in
// order.
__global__ void __launch_bounds__(256)
    bwd_dw_route(const float* __restrict__ dz, const __nv_bfloat16* __restrict__ u, int T, int N,
                 int d, float* __restrict__ dw) {
  pdl_wait();
  pdl_allow_next();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)N * d) return;
  const int j = (int)(i / d), c = (int)(i % d);
  float acc = 0.0f;
  for (int t = 0; t < T; ++t)
    acc = fmaf(dz[(size_t)t * N + j], __bfloat162float(u[(size_t)t * d + c]), acc);
  dw[i] = acc;
}

int grid_warps(int64_t warps) {
  int64_t b = (warps + 7) / 8;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b > 0 ? b : 1);
}

}  // namespace

// ------------------------------------------------- pieces shared by layers
int64_t bwd_padded_rows(const moe_shape& s) { return (int64_t)s.T * s.k + 64LL * s.N; }

BwdBufs carve_bwd(const moe_shape& s, int width, void* base) {
  Carver c(base);
  BwdBufs b;
  const int64_t R = bwd_padded_rows(s);
  b.rows = R;
  b.pad = c.take<int32_t>(s.N + 1);
  b.x = c.take<__nv_bfloat16>((size_t)R * width);
  b.dyr = c.take<__nv_bfloat16>((size_t)R * width);
  b.dyw = c.take<__nv_bfloat16>((size_t)R * width);
  b.g = c.take<__nv_bfloat16>((size_t)R * s.h);
  b.v = c.take<__nv_bfloat16>((size_t)R * s.h);
  b.H = c.take<__nv_bfloat16>((size_t)R * s.h);
  b.dG = c.take<__nv_bfloat16>((size_t)R * s.h);
  b.dV = c.take<__nv_bfloat16>((size_t)R * s.h);
  b.a = c.take<float>(R);
  b.da_part = c.take<float>((size_t)R * (s.h / 128 > 0 ? s.h / 128 : 1));
  b.dX = c.take<float>((size_t)R * width);
  b.bytes = c.used();
  return b;
}

namespace {

int launch_gather(const moe_shape& s, int width, const __nv_bfloat16* u, const __nv_bfloat16* dy,
                  const moe_layer_outputs& fwd, const BwdBufs& b, cudaStream_t st) {
  GatherParams p{};
  p.u = reinterpret_cast<const uint4*>(u);
  p.dy = reinterpret_cast<const uint4*>(dy);
  p.vec = width / 8;
  p.T = s.T;
  p.k = s.k;
  p.N = s.N;
  p.offsets = fwd.offsets;
  p.pad = b.pad;
  p.perm_tok = fwd.perm_tok;
  p.row_of = fwd.row_of;
  p.top_w = fwd.top_w;
  p.max_rows = (int)b.rows;
  p.x = reinterpret_cast<uint4*>(b.x);
  p.dyr = reinterpret_cast<uint4*>(b.dyr);
  p.dyw = reinterpret_cast<uint4*>(b.dyw);
  p.a = b.a;
  p.status = status_word();
  MOE_PREFER_SHARED((bwd_gather));
  launch_pdl(bwd_gather, dim3(grid_warps(b.rows)), dim3(256), 0, st, p);
  return launch_status();
}

}  // namespace

int experts_forward_rows(const moe_shape& s, int width, const __nv_bfloat16* u,
                         const __nv_bfloat16* Wg, const __nv_bfloat16* Wu, const moe_act& act,
                         const moe_layer_outputs& fwd, const BwdBufs& b, cudaStream_t st) {
  const int N = s.N, h = s.h;
  const int64_t R = b.rows;
  MOE_PREFER_SHARED((pad_offsets));
  launch_pdl(pad_offsets, dim3(1), dim3(32), 0, st, fwd.offsets, N, b.pad);
  int rc = launch_status();
  if (rc == MOE_OK) rc = launch_gather(s, width, u, nullptr, fwd, b, st);
  if (rc != MOE_OK) return rc;
  // the forward's pre-activations on the padded rows: G = X Wg^T, V = X Wu^T
  TcSeg sg{Wg, (int64_t)N * h, width, 0, b.x, R, width, 0};
  rc = tc_store(b.pad, (int)R, N, h, &sg, 1, b.g, MODE_STORE_BF16, h, st);
  if (rc != MOE_OK) return rc;
  TcSeg su{Wu, (int64_t)N * h, width, 0, b.x, R, width, 0};
  rc = tc_store(b.pad, (int)R, N, h, &su, 1, b.v, MODE_STORE_BF16, h, st);
  if (rc != MOE_OK) return rc;
  return bwd_hidden_rows(b.g, b.v, R * h, act, b.H, st);
}

int experts_backward_rows(const moe_shape& s, int width, const __nv_bfloat16* dy,
                          const __nv_bfloat16* Wg, const __nv_bfloat16* Wu,
                          const __nv_bfloat16* Wd, const moe_act& act,
                          const moe_layer_outputs& fwd, const BwdBufs& b, float* dw_gate,
                          float* dw_up, float* dw_down, cudaStream_t st) {
  const int N = s.N, h = s.h;
  const int64_t R = b.rows;
  int rc = launch_gather(s, width, nullptr, dy, fwd, b, st);
  if (rc != MOE_OK) return rc;
  rc = bwd_dgrad_act(b.pad, N, R, width, h, b.dyr, Wd, b.g, b.v, b.a, act, b.dG, b.dV, b.da_part,
                     st);
  if (rc != MOE_OK) return rc;
  rc = bwd_dgrad_x(b.pad, N, R, width, h, b.dG, b.dV, Wg, Wu, b.dX, st);
  if (rc != MOE_OK) return rc;
  rc = bwd_wgrad(b.pad, N, R, b.dG, h, b.x, width, dw_gate, st);
  if (rc == MOE_OK) rc = bwd_wgrad(b.pad, N, R, b.dV, h, b.x, width, dw_up, st);
  if (rc == MOE_OK) rc = bwd_wgrad(b.pad, N, R, b.dyw, width, b.H, h, dw_down, st);
  return rc;
}

int experts_backward(const moe_shape& s, int width, const __nv_bfloat16* u,
                     const __nv_bfloat16* dy, const __nv_bfloat16* Wg, const __nv_bfloat16* Wu,
                     const __nv_bfloat16* Wd, const moe_act& act, const moe_layer_outputs& fwd,
                     const BwdBufs& b, float* dw_gate, float* dw_up, float* dw_down,
                     cudaStream_t st) {
  int rc = experts_forward_rows(s, width, u, Wg, Wu, act, fwd, b, st);
  if (rc != MOE_OK) return rc;
  return experts_backward_rows(s, width, dy, Wg, Wu, Wd, act, fwd, b, dw_gate, dw_up, dw_down, st);
}

int bwd_hidden_rows(const __nv_bfloat16* g, const __nv_bfloat16* v, int64_t n,
                    const moe_act& act, __nv_bfloat16* H, cudaStream_t st) {
  const int64_t n8 = n / 8;
  if (n8 == 0) return MOE_OK;
  const int blocks = (int)std::min<int64_t>((n8 + 255) / 256, 148 * 8);
  if (act.kind == MOE_ACT_SITU_GLU) {
    MOE_PREFER_SHARED((bwd_hidden<MOE_ACT_SITU_GLU>));
    launch_pdl(bwd_hidden<MOE_ACT_SITU_GLU>, dim3(blocks), dim3(256), 0, st, g, v, n8,
               act.beta_gate, act.beta_up, H);
  } else {
    MOE_PREFER_SHARED((bwd_hidden<MOE_ACT_SWIGLU>));
    launch_pdl(bwd_hidden<MOE_ACT_SWIGLU>, dim3(blocks), dim3(256), 0, st, g, v, n8, 0.0f, 0.0f,
               H);
  }
  return launch_status();
}

int bwd_router_dz(const moe_shape& s, const moe_layer_outputs& fwd, const BwdBufs& b, float alpha,
                  const float* f, float* dz, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  DzParams p{};
  p.T = s.T;
  p.N = s.N;
  p.k = s.k;
  p.renorm = s.renorm;
  p.m_tiles = s.h / 128;
  p.top_idx = fwd.top_idx;
  p.top_w = fwd.top_w;
  p.probs = fwd.probs;
  p.row_of = fwd.row_of;
  p.offsets = fwd.offsets;
  p.pad = b.pad;
  p.da_part = b.da_part;
  p.f = f;
  p.alpha = alpha;
  p.dz = dz;
  MOE_PREFER_SHARED((bwd_dz));
  launch_pdl(bwd_dz, dim3((s.T + 7) / 8), dim3(256), 0, st, p);
  return launch_status();
}

int bwd_token_sum(const moe_shape& s, int width, const moe_layer_outputs& fwd, const BwdBufs* b,
                  const float* dz, const float* w_route, float* out, bool add, cudaStream_t st) {
  if (s.T == 0) return MOE_OK;
  DuParams p{};
  p.T = s.T;
  p.N = s.N;
  p.k = s.k;
  p.d = width;
  p.top_idx = fwd.top_idx;
  p.row_of = fwd.row_of;
  p.offsets = fwd.offsets;
  p.pad = b ? b->pad : nullptr;
  p.dX = b ? b->dX : nullptr;
  p.dz = dz;
  p.w_route = w_route;
  p.du = out;
  p.add = add ? 1 : 0;
  MOE_PREFER_SHARED((bwd_du));
  launch_pdl(bwd_du, dim3(grid_warps(s.T)), dim3(256), 0, st, p);
  return launch_status();
}

int bwd_router_wgrad(const float* dz, const __nv_bfloat16* u, int T, int N, int d, float* dw,
                     cudaStream_t st) {
  const int64_t n = (int64_t)N * d;
  if (n == 0) return MOE_OK;
  MOE_PREFER_SHARED((bwd_dw_route));
  launch_pdl(bwd_dw_route, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, dz, u, T, N, d,
             dw);
  return launch_status();
}

bool bwd_act_ok(const moe_act& a) {
  return a.kind == MOE_ACT_SWIGLU ||
         (a.kind == MOE_ACT_SITU_GLU && a.beta_gate > 0.0f && a.beta_up > 0.0f);
}

}  // namespace moe

extern "C" size_t moe_layer_bwd_workspace_bytes(const moe_shape* shape) {
  using namespace moe;
  if (!shape_ok(shape) || shape->h <= 0 || shape->h % 128 != 0 || shape->d % 128 != 0) return 0;
  return carve_bwd(*shape, shape->d, nullptr).bytes;
}

extern "C" int moe_layer_bwd(const moe_shape* shape, const moe_layer_weights* w, const void* u,
                             const void* dy, const moe_layer_outputs* fwd, float alpha,
                             const float* f, const moe_layer_grads* grads, void* ws,
                             size_t ws_bytes, void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || shape->h <= 0 || shape->h % 128 != 0 || shape->d % 128 != 0 || !w ||
      !fwd || !grads)
    return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (w->w_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!bwd_act_ok(w->act)) return MOE_ERR_INVALID_ARG;
  if (!w->w_route || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (!fwd->top_idx || !fwd->top_w || !fwd->probs || !fwd->row_of || !fwd->offsets ||
      !fwd->perm_tok)
    return MOE_ERR_INVALID_ARG;
  if (!grads->du || !grads->dz || !grads->dw_gate || !grads->dw_up || !grads->dw_down)
    return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (!u || !dy)) return MOE_ERR_INVALID_ARG;
  const void* al[] = {u, dy, w->w_route, w->w_gate, w->w_up, w->w_down, grads->du,
                      grads->dw_gate, grads->dw_up, grads->dw_down, grads->dw_route};
  for (const void* q : al)
    if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
  BwdBufs b = carve_bwd(s, s.d, ws);
  if (!ws || ws_bytes < b.bytes) return MOE_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  const auto* U = static_cast<const __nv_bfloat16*>(u);
  int rc = experts_backward(s, s.d, U, static_cast<const __nv_bfloat16*>(dy),
                            static_cast<const __nv_bfloat16*>(w->w_gate),
                            static_cast<const __nv_bfloat16*>(w->w_up),
                            static_cast<const __nv_bfloat16*>(w->w_down), w->act, *fwd, b,
                            grads->dw_gate, grads->dw_up, grads->dw_down, st);
  if (rc == MOE_OK) rc = bwd_router_dz(s, *fwd, b, alpha, f, grads->dz, st);
  // du = the kept slots' expert input gradients + sum_j dz_j W_route[j]
  if (rc == MOE_OK)
    rc = bwd_token_sum(s, s.d, *fwd, &b, grads->dz, w->w_route, grads->du, false, st);
  if (rc == MOE_OK && grads->dw_route)
    rc = bwd_router_wgrad(grads->dz, U, s.T, s.N, s.d, grads->dw_route, st);
  return rc;
}
