// The LatentMoE layer backward ("Stable LatentMoE interactive demo document":
// width separation, RMSNorm before the up-projection, SiTU-GLU routed
// experts, plain SwiGLU shared experts; the tutorial "Mixture of Experts
// MoE: how sparse activation saves compute" §3.1-§3.2 for the routed layer),
// with the selected sets held fixed, for L = sum_t dy_t . y_t:
//   y = W_upp m^ + sum_j S_j(x),  m^ = m / r,  r = sqrt(mean(m^2) + eps),
//   m = sum_s a_s E_s(x_l),  x_l = W_dp x,  z = W_route x (+ b)
// Steps (bf16 operands, fp32 accumulation and gradients):
//   recompute x_l and the routed forward rows, m = sum of the kept rows a F
//   dm^ = dy W_upp,  dW_upp = dy^T m^
//   dm = (dm^ - m^ mean(dm^ . m^)) / r                       (RMSNorm)
//   the routed experts' backward with upstream dm on inputs x_l -> dx_l
//   rows, routed weight gradients, dz (softmax / renormalisation backward)
//   dx = dx_l W_dp + sum_j dz_j W_route[j] + sum_j dS_j/dx,
//   dW_dp = dx_l^T x,  dW_route = dz^T x,  the shared experts' gradients
#include <algorithm>

#include "bwd.cuh"

namespace moe {
namespace {

int rows_grid(int64_t warps) {
  int64_t b = (warps + 7) / 8;
  if (b > 148 * 16) b = 148 * 16;
  return (int)(b > 0 ? b : 1);
}

// dst [T_pad][w] = src [T][w] rows, zero rows beyond T (16-byte vectors).
__global__ void __launch_bounds__(256)
    pad_rows_bf16(const uint4* __restrict__ src, int T, int T_pad, int vec,
                  uint4* __restrict__ dst) {
  pdl_wait();
  pdl_allow_next();
  const int64_t n = (int64_t)T_pad * vec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = i / vec < T ? src[i] : make_uint4(0, 0, 0, 0);
}

// n copies of src [rows][vec] one after another.
__global__ void __launch_bounds__(256)
    repeat_rows(const uint4* __restrict__ src, int64_t count, int n, uint4* __restrict__ dst) {
  pdl_wait();
  pdl_allow_next();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count * n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i % count];
}

// Group offsets {0, rows, 2 rows, ...} and ones, for the dense layers read as
// groups.
__global__ void fill_groups(int32_t* offsets, int G, int rows, float* ones, int64_t n_ones) {
  pdl_wait();
  pdl_allow_next();
  for (int g = threadIdx.x; g <= G; g += blockDim.x) offsets[g] = g * rows;
  for (int64_t i = threadIdx.x; i < n_ones; i += blockDim.x) ones[i] = 1.0f;
}

// One warp per token: r = sqrt(mean(m^2) + eps), m^ = m / r as bf16 (the
// forward's rounding), inv_r.
__global__ void __launch_bounds__(256)
    rms_forward(const float* __restrict__ m, int T, int T_pad, int l, float eps,
                __nv_bfloat16* __restrict__ mh, float* __restrict__ inv_r) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T_pad;
       t += (gridDim.x * blockDim.x) >> 5) {
    if (t >= T) {  // padding rows: zero, so the weight-gradient sums see 0 x 0
      for (int c = lane; c < l; c += 32) mh[(size_t)t * l + c] = __float2bfloat16_rn(0.0f);
      continue;
    }
    const float* x = m + (size_t)t * l;
    float ss = 0.0f;
    for (int c = lane; c < l; c += 32) ss = fmaf(x[c], x[c], ss);
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)l + eps);
    for (int c = lane; c < l; c += 32) mh[(size_t)t * l + c] = __float2bfloat16_rn(x[c] * inv);
    if (lane == 0) inv_r[t] = inv;
  }
}

// One warp per token: dm = (dm^ - m^ mean(dm^ . m^)) / r with m^ = m / r in
// fp32; bf16 out.
__global__ void __launch_bounds__(256)
    rms_backward(const float* __restrict__ m, const float* __restrict__ dmh,
                 const float* __restrict__ inv_r, int T, int l, __nv_bfloat16* __restrict__ dm) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T;
       t += (gridDim.x * blockDim.x) >> 5) {
    const float inv = inv_r[t];
    const float* x = m + (size_t)t * l;
    const float* g = dmh + (size_t)t * l;
    float dot = 0.0f;
    for (int c = lane; c < l; c += 32) dot = fmaf(g[c], x[c] * inv, dot);
    for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float mean = dot / (float)l;
    for (int c = lane; c < l; c += 32)
      dm[(size_t)t * l + c] = __float2bfloat16_rn((g[c] - x[c] * inv * mean) * inv);
  }
}

// dst [T_pad][w] bf16 from src fp32 [T][w], zero rows beyond T.
__global__ void __launch_bounds__(256)
    to_bf16_padded(const float* __restrict__ src, int T, int T_pad, int w,
                   __nv_bfloat16* __restrict__ dst) {
  pdl_wait();
  pdl_allow_next();
  const int64_t n = (int64_t)T_pad * w;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(i / w < T ? src[i] : 0.0f);
}

// out [T][w] = a [T][w] + sum_j parts[j * stride + t], n_parts blocks of
// `stride` rows, in that order.
__global__ void __launch_bounds__(256)
    sum_rows(const float* __restrict__ a, const float* __restrict__ parts, int n_parts,
             int64_t stride, int T, int w, float* __restrict__ out) {
  pdl_wait();
  pdl_allow_next();
  const int64_t n = (int64_t)T * w;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = a[i];
    for (int j = 0; j < n_parts; ++j) v += parts[(size_t)j * stride * w + i];
    out[i] = v;
  }
}

int flat_grid(int64_t n) {
  int64_t b = (n + 255) / 256;
  if (b > 148 * 8) b = 148 * 8;
  return (int)(b > 0 ? b : 1);
}

struct LatentBwdBufs {
  BwdBufs r;                 // routed experts (width l)
  int64_t T_pad;
  __nv_bfloat16 *x_pad, *dy_pad, *x_l, *mh, *dm, *dxl;
  float *m, *inv_r, *dmh, *dxl_f, *dx_a;
  int32_t* grp1;             // {0, T_pad}
  int32_t* grpn;             // {0, T_pad, 2 T_pad, ...}
  float* ones;               // [n * T_pad]
  __nv_bfloat16 *x2, *dy2, *sg, *sv, *sH, *sdG, *sdV;
  float *s_part, *sdX;
  size_t bytes;
};

LatentBwdBufs carve_latent_bwd(const moe_shape& s, const moe_latent_weights& lw, void* base) {
  LatentBwdBufs b;
  const int64_t T_pad = ((int64_t)s.T + 63) / 64 * 64;
  const int l = lw.latent, d = s.d, n = lw.n_shared, sh = lw.shared_hidden > 0 ? lw.shared_hidden : 1;
  b.T_pad = T_pad;
  Carver c(base);
  const size_t r_bytes = carve_bwd(s, l, nullptr).bytes;
  char* r_base = c.take<char>(r_bytes);
  b.r = carve_bwd(s, l, r_base);
  b.x_pad = c.take<__nv_bfloat16>((size_t)T_pad * d);
  b.dy_pad = c.take<__nv_bfloat16>((size_t)T_pad * d);
  b.x_l = c.take<__nv_bfloat16>((size_t)T_pad * l);
  b.mh = c.take<__nv_bfloat16>((size_t)T_pad * l);
  b.dm = c.take<__nv_bfloat16>((size_t)T_pad * l);
  b.dxl = c.take<__nv_bfloat16>((size_t)T_pad * l);
  b.m = c.take<float>((size_t)T_pad * l);
  b.inv_r = c.take<float>(T_pad);
  b.dmh = c.take<float>((size_t)T_pad * l);
  b.dxl_f = c.take<float>((size_t)T_pad * l);
  b.dx_a = c.take<float>((size_t)T_pad * d);
  b.grp1 = c.take<int32_t>(2);
  b.grpn = c.take<int32_t>(n + 1);
  b.ones = c.take<float>((size_t)(n > 0 ? n : 1) * T_pad);
  const size_t rows_n = (size_t)(n > 0 ? n : 1) * T_pad;
  b.x2 = c.take<__nv_bfloat16>(rows_n * d);
  b.dy2 = c.take<__nv_bfloat16>(rows_n * d);
  b.sg = c.take<__nv_bfloat16>(rows_n * sh);
  b.sv = c.take<__nv_bfloat16>(rows_n * sh);
  b.sH = c.take<__nv_bfloat16>(rows_n * sh);
  b.sdG = c.take<__nv_bfloat16>(rows_n * sh);
  b.sdV = c.take<__nv_bfloat16>(rows_n * sh);
  b.s_part = c.take<float>(rows_n * (sh / 128 > 0 ? sh / 128 : 1));
  b.sdX = c.take<float>(rows_n * d);
  b.bytes = c.used();
  if (!base) b.r = BwdBufs{};
  return b;
}

bool latent_bwd_ok(const moe_shape* s, const moe_latent_weights* lw) {
  if (!shape_ok(s) || !lw) return false;
  const int l = lw->latent;
  if (l <= 0 || l % 128 != 0 || s->d % 128 != 0 || s->h <= 0 || s->h % 128 != 0) return false;
  if (lw->n_shared < 0 || lw->n_shared > 2) return false;
  if (lw->n_shared > 0 && (lw->shared_hidden <= 0 || lw->shared_hidden % 128 != 0)) return false;
  return lw->rms_eps >= 0.0f;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_latent_bwd_workspace_bytes(const moe_shape* shape,
                                                 const moe_latent_weights* lw) {
  if (!moe::latent_bwd_ok(shape, lw)) return 0;
  return moe::carve_latent_bwd(*shape, *lw, nullptr).bytes;
}

extern "C" int moe_latent_bwd(const moe_shape* shape, const moe_layer_weights* w,
                              const moe_latent_weights* lw, const void* x, const void* dy,
                              const moe_layer_outputs* fwd, const moe_latent_grads* g, void* ws,
                              size_t ws_bytes, void* stream) {
  using namespace moe;
  if (!latent_bwd_ok(shape, lw) || !w || !fwd || !g) return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (w->w_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!bwd_act_ok(w->act)) return MOE_ERR_INVALID_ARG;
  if (!w->w_route || !w->w_gate || !w->w_up || !w->w_down || !lw->w_down_proj || !lw->w_up_proj)
    return MOE_ERR_INVALID_ARG;
  const int n = lw->n_shared;
  if (n > 0 && (!lw->shared_gate || !lw->shared_up || !lw->shared_down)) return MOE_ERR_INVALID_ARG;
  if (!fwd->top_idx || !fwd->top_w || !fwd->probs || !fwd->row_of || !fwd->offsets ||
      !fwd->perm_tok)
    return MOE_ERR_INVALID_ARG;
  if (!g->dx || !g->dz || !g->dw_gate || !g->dw_up || !g->dw_down || !g->dw_dp || !g->dw_upp)
    return MOE_ERR_INVALID_ARG;
  if (n > 0 && (!g->dsh_gate || !g->dsh_up || !g->dsh_down)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (!x || !dy)) return MOE_ERR_INVALID_ARG;
  const void* al[] = {x, dy, w->w_gate, w->w_up, w->w_down, lw->w_down_proj, lw->w_up_proj,
                      lw->shared_gate, lw->shared_up, lw->shared_down, g->dx, g->dw_route,
                      g->dw_gate, g->dw_up, g->dw_down, g->dw_dp, g->dw_upp, g->dsh_gate,
                      g->dsh_up, g->dsh_down};
  for (const void* q : al)
    if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
  LatentBwdBufs b = carve_latent_bwd(s, *lw, ws);
  if (!ws || ws_bytes < b.bytes) return MOE_ERR_WORKSPACE;
  if (s.T == 0) return MOE_OK;
  cudaStream_t st = as_stream(stream);
  const int d = s.d, l = lw->latent, T = s.T, sh = lw->shared_hidden;
  const int Tp = (int)b.T_pad;
  const auto* X = static_cast<const __nv_bfloat16*>(x);
  const auto* Wg = static_cast<const __nv_bfloat16*>(w->w_gate);
  const auto* Wu = static_cast<const __nv_bfloat16*>(w->w_up);
  const auto* Wd = static_cast<const __nv_bfloat16*>(w->w_down);
  const auto* Wdp = static_cast<const __nv_bfloat16*>(lw->w_down_proj);
  const auto* Wupp = static_cast<const __nv_bfloat16*>(lw->w_up_proj);
  int rc;
#define MOE_LAUNCH(kernel, grid, ...)                                   \
  do {                                                                  \
    MOE_PREFER_SHARED((kernel));                                        \
    launch_pdl(kernel, dim3(grid), dim3(256), 0, st, __VA_ARGS__);      \
    if ((rc = launch_status()) != MOE_OK) return rc;                    \
  } while (0)

  // padded copies of x and dy, group tables, ones
  MOE_LAUNCH(pad_rows_bf16, flat_grid((int64_t)Tp * d / 8), static_cast<const uint4*>(x), T, Tp,
             d / 8, reinterpret_cast<uint4*>(b.x_pad));
  MOE_LAUNCH(pad_rows_bf16, flat_grid((int64_t)Tp * d / 8), static_cast<const uint4*>(dy), T, Tp,
             d / 8, reinterpret_cast<uint4*>(b.dy_pad));
  MOE_LAUNCH(fill_groups, 1, b.grp1, 1, Tp, b.ones, (int64_t)0);
  if (n > 0) MOE_LAUNCH(fill_groups, 1, b.grpn, n, Tp, b.ones, (int64_t)n * Tp);

  // x_l = bf16(W_dp x) on the padded rows (zero rows stay zero)
  {
    TcSeg seg{Wdp, l, d, 0, b.x_pad, Tp, d, 0};
    rc = tc_store(b.grp1, Tp, 1, l, &seg, 1, b.x_l, MODE_STORE_BF16, l, st);
    if (rc != MOE_OK) return rc;
  }
  // the routed forward rows and m = sum of the kept slots' a F rows (fp32)
  rc = experts_forward_rows(s, l, b.x_l, Wg, Wu, w->act, *fwd, b.r, st);
  if (rc != MOE_OK) return rc;
  {
    TcSeg seg{Wd, (int64_t)s.N * l, s.h, 0, b.r.H, b.r.rows, s.h, 0};
    rc = tc_store(b.r.pad, (int)b.r.rows, s.N, l, &seg, 1, b.r.dX, MODE_STORE_F32, l, st, nullptr,
                  b.r.a);
    if (rc != MOE_OK) return rc;
    rc = bwd_token_sum(s, l, *fwd, &b.r, nullptr, nullptr, b.m, false, st);
    if (rc != MOE_OK) return rc;
  }
  MOE_LAUNCH(rms_forward, rows_grid(Tp), b.m, T, Tp, l, lw->rms_eps, b.mh, b.inv_r);
  // dm^ = dy W_upp (W_upp [d][l] read MN-major), dW_upp = dy^T m^
  rc = bwd_dgrad_plain(b.grp1, 1, Tp, d, l, b.dy_pad, Wupp, b.dmh, st);
  if (rc != MOE_OK) return rc;
  rc = bwd_wgrad(b.grp1, 1, Tp, b.dy_pad, d, b.mh, l, g->dw_upp, st);
  if (rc != MOE_OK) return rc;
  // RMSNorm backward -> dm (bf16, the routed experts' upstream gradient)
  MOE_LAUNCH(rms_backward, rows_grid(T), b.m, b.dmh, b.inv_r, T, l, b.dm);
  // the routed experts' backward with upstream dm on x_l
  rc = experts_backward_rows(s, l, b.dm, Wg, Wu, Wd, w->act, *fwd, b.r, g->dw_gate, g->dw_up,
                             g->dw_down, st);
  if (rc == MOE_OK) rc = bwd_router_dz(s, *fwd, b.r, 0.0f, nullptr, g->dz, st);
  if (rc != MOE_OK) return rc;
  // dx_l = sum of the kept slots' input-gradient rows; dx = dx_l W_dp; dW_dp
  rc = bwd_token_sum(s, l, *fwd, &b.r, nullptr, nullptr, b.dxl_f, false, st);
  if (rc != MOE_OK) return rc;
  MOE_LAUNCH(to_bf16_padded, flat_grid((int64_t)Tp * l), b.dxl_f, T, Tp, l, b.dxl);
  rc = bwd_dgrad_plain(b.grp1, 1, Tp, l, d, b.dxl, Wdp, b.dx_a, st);
  if (rc == MOE_OK) rc = bwd_wgrad(b.grp1, 1, Tp, b.dxl, l, b.x_pad, d, g->dw_dp, st);
  if (rc != MOE_OK) return rc;
  // the router on x: dx += sum_j dz_j W_route[j], dW_route = dz^T x
  rc = bwd_token_sum(s, d, *fwd, nullptr, g->dz, w->w_route, b.dx_a, true, st);
  if (rc == MOE_OK && g->dw_route) rc = bwd_router_wgrad(g->dz, X, T, s.N, d, g->dw_route, st);
  if (rc != MOE_OK) return rc;
  // the shared experts (plain SwiGLU on x), as n groups over copies of x
  if (n > 0) {
    const int64_t R2 = (int64_t)n * Tp;
    const auto* Sg = static_cast<const __nv_bfloat16*>(lw->shared_gate);
    const auto* Su = static_cast<const __nv_bfloat16*>(lw->shared_up);
    const auto* Sd = static_cast<const __nv_bfloat16*>(lw->shared_down);
    MOE_LAUNCH(repeat_rows, flat_grid(R2 * d / 8), reinterpret_cast<const uint4*>(b.x_pad),
               (int64_t)Tp * d / 8, n, reinterpret_cast<uint4*>(b.x2));
    MOE_LAUNCH(repeat_rows, flat_grid(R2 * d / 8), reinterpret_cast<const uint4*>(b.dy_pad),
               (int64_t)Tp * d / 8, n, reinterpret_cast<uint4*>(b.dy2));
    TcSeg sgs{Sg, (int64_t)n * sh, d, 0, b.x2, R2, d, 0};
    rc = tc_store(b.grpn, (int)R2, n, sh, &sgs, 1, b.sg, MODE_STORE_BF16, sh, st);
    if (rc != MOE_OK) return rc;
    TcSeg sus{Su, (int64_t)n * sh, d, 0, b.x2, R2, d, 0};
    rc = tc_store(b.grpn, (int)R2, n, sh, &sus, 1, b.sv, MODE_STORE_BF16, sh, st);
    if (rc != MOE_OK) return rc;
    const moe_act swiglu{MOE_ACT_SWIGLU, 0.0f, 0.0f};
    rc = bwd_hidden_rows(b.sg, b.sv, R2 * sh, swiglu, b.sH, st);
    if (rc == MOE_OK)
      rc = bwd_dgrad_act(b.grpn, n, R2, d, sh, b.dy2, Sd, b.sg, b.sv, b.ones, swiglu, b.sdG,
                         b.sdV, b.s_part, st);
    if (rc == MOE_OK) rc = bwd_dgrad_x(b.grpn, n, R2, d, sh, b.sdG, b.sdV, Sg, Su, b.sdX, st);
    if (rc == MOE_OK) rc = bwd_wgrad(b.grpn, n, R2, b.sdG, sh, b.x2, d, g->dsh_gate, st);
    if (rc == MOE_OK) rc = bwd_wgrad(b.grpn, n, R2, b.sdV, sh, b.x2, d, g->dsh_up, st);
    if (rc == MOE_OK) rc = bwd_wgrad(b.grpn, n, R2, b.dy2, d, b.sH, sh, g->dsh_down, st);
    if (rc != MOE_OK) return rc;
  }
  // dx = the routed and router part + the shared experts' parts, fixed order
  MOE_LAUNCH(sum_rows, flat_grid((int64_t)T * d), b.dx_a, b.sdX, n, (int64_t)Tp, T, d, g->dx);
#undef MOE_LAUNCH
  return MOE_OK;
}
