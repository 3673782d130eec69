// LatentMoE layer forward ("Stable LatentMoE interactive demo document"):
// routed experts live in a narrower latent space, shared experts at full
// width, RMSNorm after the routed aggregation and before the up-projection,
// SiTU-GLU soft caps on the routed experts' gate and up.
//
//   z = W_route x (+b) on the full-width x      -> top-k, a   (router reading)
//   x_l = W_dp x                  [T][l]  bf16   tcgen05 GEMM, one group
//   m = sum_s a_s E_s(x_l)        [T][l]  fp32   permute, gather, grouped
//                                                gate/up (SiTU-GLU) + down,
//                                                combine
//   m^ = m / sqrt(mean(m^2) + eps)          bf16   rmsnorm_rows
//   H_j = SwiGLU gate/up of shared expert j on x   tcgen05 GEMM, n_shared groups
//   y = W_upp m^ + sum_j W_down,j H_j   [T][d]  bf16   one tcgen05 GEMM over
//                                                1 + n_shared K-segments
#include "common.cuh"

namespace moe {

namespace {

// One warp per row: sum of squares in fp32, then x / sqrt(mean + eps) -> bf16.
__global__ void __launch_bounds__(256)
    rmsnorm_rows(const float* __restrict__ m, int rows, int cols, float eps,
                 __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_allow_next();
  const int lane = threadIdx.x & 31;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += (gridDim.x * blockDim.x) >> 5) {
    const float4* x = reinterpret_cast<const float4*>(m + (size_t)r * cols);
    float ss = 0.0f;
    for (int c = lane; c < cols / 4; c += 32) {
      const float4 v = x[c];
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)cols + eps);
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(out + (size_t)r * cols);
    for (int c = lane; c < cols / 4; c += 32) {
      const float4 v = x[c];
      o2[2 * c] = __floats2bfloat162_rn(v.x * inv, v.y * inv);
      o2[2 * c + 1] = __floats2bfloat162_rn(v.z * inv, v.w * inv);
    }
  }
}

struct LatentBufs {
  int32_t* top_idx;
  float* top_w;
  float* probs;
  float* logits;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm_tok;
  int32_t* row_of;
  int32_t* overflow;
  int32_t* totals;
  void* permute_ws;
  __nv_bfloat16* x_l;
  __nv_bfloat16* x_rows;  // E4M3 experts: the gathered codes of x_l (1 byte each)
  float* x_scale;         // E4M3 experts: one scale per gathered row
  __nv_bfloat16* H;       // E4M3 experts: H as codes
  float* y_rows;  // fp32 rows a * E(x_l)
  float* row_w;   // combine weight of each grouped row
  float* m;
  __nv_bfloat16* m_hat;
  __nv_bfloat16* H_sh;
  void* stats_ws;
  size_t bytes;
};

LatentBufs carve_latent(const moe_shape& s, const moe_latent_weights& lw, void* base) {
  Carver c(base);
  LatentBufs b;
  const size_t Tk = (size_t)s.T * s.k, l = lw.latent;
  b.top_idx = c.take<int32_t>(Tk);
  b.top_w = c.take<float>(Tk);
  b.probs = c.take<float>((size_t)s.T * s.N);
  b.logits = c.take<float>((size_t)s.T * s.N);
  b.counts = c.take<int32_t>(s.N);
  b.offsets = c.take<int32_t>(s.N + 1);
  b.perm_tok = c.take<int32_t>(Tk);
  b.row_of = c.take<int32_t>(Tk);
  b.overflow = c.take<int32_t>(s.N);
  b.totals = c.take<int32_t>(4);
  b.permute_ws = c.take<char>(permute_ws_bytes(s));
  b.x_l = c.take<__nv_bfloat16>((size_t)s.T * l);
  b.x_rows = c.take<__nv_bfloat16>(Tk * l);
  b.x_scale = c.take<float>(Tk);
  b.H = c.take<__nv_bfloat16>(Tk * s.h);
  b.y_rows = c.take<float>(Tk * l);
  b.row_w = c.take<float>(Tk);
  b.m = c.take<float>((size_t)s.T * l);
  b.m_hat = c.take<__nv_bfloat16>((size_t)s.T * l);
  b.H_sh = c.take<__nv_bfloat16>((size_t)s.T * (lw.n_shared > 0 ? lw.n_shared : 1) *
                                 (lw.shared_hidden > 0 ? lw.shared_hidden : 1));
  b.stats_ws = c.take<char>(aux_stats_ws_bytes(s.N));
  b.bytes = c.used();
  return b;
}

bool latent_ok(const moe_shape* s, const moe_latent_weights* lw) {
  if (!shape_ok(s) || !lw) return false;
  const int l = lw->latent;
  if (l <= 0 || l % 128 != 0 || s->d % 128 != 0 || s->h % 64 != 0) return false;
  if (lw->n_shared < 0 || lw->n_shared > 2) return false;
  if (lw->n_shared > 0 && (lw->shared_hidden <= 0 || lw->shared_hidden % 64 != 0)) return false;
  if (!(lw->rms_eps >= 0.0f)) return false;
  return true;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_latent_workspace_bytes(const moe_shape* shape,
                                             const moe_latent_weights* lw) {
  if (!moe::latent_ok(shape, lw)) return 0;
  return moe::carve_latent(*shape, *lw, nullptr).bytes;
}

namespace moe {
namespace {

// The layer with bf16 routed experts (e4m3 == nullptr) or E4M3 ones.
int latent_forward(const moe_shape* shape, const moe_layer_weights* w,
                   const moe_e4m3_scales* e4m3, const moe_latent_weights* lw, const void* x,
                   void* y, const moe_layer_outputs* out, void* ws, size_t ws_bytes,
                   void* stream) {
  if (!latent_ok(shape, lw) || !w) return MOE_ERR_INVALID_ARG;
  if (w->w_dtype != (e4m3 ? MOE_E4M3 : MOE_BF16)) return MOE_ERR_UNSUPPORTED;
  if (e4m3 && (!e4m3->gate_scale || !e4m3->up_scale || !e4m3->down_scale))
    return MOE_ERR_INVALID_ARG;
  if (e4m3 && (lw->latent % 128 != 0 || shape->h % 128 != 0)) return MOE_ERR_UNSUPPORTED;
  if (w->act.kind != MOE_ACT_SWIGLU &&
      !(w->act.kind == MOE_ACT_SITU_GLU && w->act.beta_gate > 0.0f && w->act.beta_up > 0.0f))
    return MOE_ERR_INVALID_ARG;
  if (!w->w_route || !w->w_gate || !w->w_up || !w->w_down || !lw->w_down_proj ||
      !lw->w_up_proj)
    return MOE_ERR_INVALID_ARG;
  if (lw->n_shared > 0 && (!lw->shared_gate || !lw->shared_up || !lw->shared_down))
    return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (s.T > 0 && (!x || !y)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, y, w->w_route, w->w_gate, w->w_up, w->w_down, lw->w_down_proj,
                        lw->w_up_proj, lw->shared_gate, lw->shared_up, lw->shared_down};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  LatentBufs b = carve_latent(s, *lw, ws);
  if (!ws || ws_bytes < b.bytes) return MOE_ERR_WORKSPACE;
  if (s.T == 0) return MOE_OK;
  moe_layer_outputs o{};
  if (out) o = *out;
  const bool want_stats = o.f || o.P || o.n_sum_fP;
  int32_t* top_idx = o.top_idx ? o.top_idx : b.top_idx;
  float* top_w = o.top_w ? o.top_w : b.top_w;
  float* probs = o.probs ? o.probs : (want_stats ? b.probs : nullptr);
  int32_t* counts = o.counts ? o.counts : b.counts;
  int32_t* offsets = o.offsets ? o.offsets : b.offsets;
  int32_t* perm_tok = o.perm_tok ? o.perm_tok : b.perm_tok;
  int32_t* row_of = o.row_of ? o.row_of : b.row_of;
  int32_t* overflow = o.overflow ? o.overflow : b.overflow;
  int32_t* totals = o.totals ? o.totals : b.totals;
  cudaStream_t st = as_stream(stream);
  const int l = lw->latent, Tk = s.T * s.k;
  const auto* X = static_cast<const __nv_bfloat16*>(x);

  int rc = launch_route(s, x, MOE_BF16, w->w_route, w->bias, top_idx, top_w, probs, b.logits,
                        nullptr, st);
  if (rc == MOE_OK && want_stats)
    rc = launch_aux_stats(s.T, s.N, s.k, probs, top_idx, o.f, o.P, o.n_sum_fP, nullptr,
                          b.stats_ws, st);
  if (rc == MOE_OK)
    rc = launch_permute(s, top_idx, counts, offsets, perm_tok, row_of, overflow, totals,
                        b.permute_ws, st, top_w, b.row_w);
  if (rc != MOE_OK) return rc;
  // x_l = W_dp x (width separation: routed experts work in l < d)
  {
    TcSeg seg{lw->w_down_proj, l, s.d, 0, X, s.T, s.d, 0};
    rc = tc_store(nullptr, s.T, 1, l, &seg, 1, b.x_l, MODE_STORE_BF16, l, st);
    if (rc != MOE_OK) return rc;
  }
  if (e4m3) {
    // E4M3 experts: x_l quantised per token while it is gathered; gate/up
    // with the row scales, H stored as E4M3 codes; down with its row scales
    TcF8 gu{{e4m3->gate_scale, e4m3->up_scale}, b.x_scale};
    TcF8 dn{{e4m3->down_scale, nullptr}, b.row_w};
    rc = launch_quant_gather_e4m3(s, l, b.x_l, perm_tok, offsets,
                                  reinterpret_cast<uint8_t*>(b.x_rows), b.x_scale, st);
    if (rc == MOE_OK)
      rc = tc_gateup(offsets, Tk, s.N, b.x_rows, Tk, l, w->w_gate, w->w_up, s.h, w->act, b.H, s.h,
                     0, st, &gu);
    if (rc != MOE_OK) return rc;
    TcSeg seg{w->w_down, (int64_t)s.N * l, s.h, 0, b.H, Tk, s.h, 0};
    rc = tc_store(offsets, Tk, s.N, l, &seg, 1, b.y_rows, MODE_STORE_F32, l, st, &dn);
    if (rc != MOE_OK) return rc;
  } else {
    rc = launch_gather(s, l, b.x_l, MOE_BF16, perm_tok, offsets, b.x_rows, st);
    if (rc != MOE_OK) return rc;
    rc = tc_gateup(offsets, Tk, s.N, b.x_rows, Tk, l, w->w_gate, w->w_up, s.h, w->act, b.H, s.h,
                   0, st);
    if (rc != MOE_OK) return rc;
    TcSeg seg{w->w_down, (int64_t)s.N * l, s.h, 0, b.H, Tk, s.h, 0};
    rc = tc_store(offsets, Tk, s.N, l, &seg, 1, b.y_rows, MODE_STORE_F32, l, st, nullptr,
                  b.row_w);
    if (rc != MOE_OK) return rc;
  }
  // the down GEMMs stored rows a * E(x_l): the combine adds them
  rc = launch_combine_weighted(s, l, b.y_rows, row_of, b.m, MOE_F32, st);
  if (rc != MOE_OK) return rc;
  {
    int blocks = (s.T + 7) / 8;
    if (blocks > 148 * 16) blocks = 148 * 16;
    MOE_PREFER_SHARED((rmsnorm_rows));
    launch_pdl(rmsnorm_rows, dim3(blocks), dim3(256), 0, st, b.m, s.T, l, lw->rms_eps, b.m_hat);
    rc = launch_status();
    if (rc != MOE_OK) return rc;
  }
  const int nsh = lw->n_shared, sh = lw->shared_hidden;
  if (nsh > 0) {
    moe_act swiglu{MOE_ACT_SWIGLU, 0.0f, 0.0f};
    rc = tc_gateup(nullptr, s.T, nsh, X, s.T, s.d,
                   static_cast<const __nv_bfloat16*>(lw->shared_gate),
                   static_cast<const __nv_bfloat16*>(lw->shared_up), sh, swiglu, b.H_sh, nsh * sh,
                   sh, st);
    if (rc != MOE_OK) return rc;
  }
  // y = W_upp m^ + sum_j W_down,j H_j: one accumulator over 1 + n_shared segments
  TcSeg segs[3];
  segs[0] = TcSeg{lw->w_up_proj, s.d, l, 0, b.m_hat, s.T, l, 0};
  for (int j = 0; j < nsh; ++j)
    segs[1 + j] = TcSeg{lw->shared_down, (int64_t)nsh * s.d, sh, j * s.d, b.H_sh, s.T, nsh * sh,
                        j * sh};
  return tc_store(nullptr, s.T, 1, s.d, segs, 1 + nsh, y, MODE_STORE_BF16, s.d, st);
}

}  // namespace
}  // namespace moe

extern "C" int moe_latent_fwd(const moe_shape* shape, const moe_layer_weights* w,
                              const moe_latent_weights* lw, const void* x, void* y,
                              const moe_layer_outputs* out, void* ws, size_t ws_bytes,
                              void* stream) {
  return moe::latent_forward(shape, w, nullptr, lw, x, y, out, ws, ws_bytes, stream);
}

extern "C" int moe_latent_fwd_e4m3(const moe_shape* shape, const moe_layer_weights* w,
                                   const moe_e4m3_scales* scales, const moe_latent_weights* lw,
                                   const void* x, void* y, const moe_layer_outputs* out, void* ws,
                                   size_t ws_bytes, void* stream) {
  if (!scales) return MOE_ERR_INVALID_ARG;
  return moe::latent_forward(shape, w, scales, lw, x, y, out, ws, ws_bytes, stream);
}
