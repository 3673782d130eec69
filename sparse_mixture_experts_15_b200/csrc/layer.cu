// The expert FFN entry point and the whole-layer forward: router -> aux
// statistics -> permutation -> gather -> grouped experts -> weighted combine
// (tutorial "Mixture of Experts MoE: how sparse activation saves compute",
// §3.1-§3.8).  Every step is one of this library's kernels, launched in order
// on the caller's stream; nothing is read back to the host.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

struct LayerBufs {
  float* logits;
  int32_t* top_idx;
  float* top_w;
  float* probs;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm_tok;
  int32_t* row_of;
  int32_t* overflow;
  int32_t* totals;
  void* permute_ws;
  void* x_rows;
  void* ffn_ws;
  float* y_rows;  // bf16 layers: fp32 rows a * F(u)
  float* row_w;   // combine weight of each grouped row
  void* stats_ws;
  void* rd_ws;
  size_t bytes;
};

bool ffn_supported(const moe_shape& s, int32_t width, int32_t dtype) {
  if (dtype == MOE_F32) return (size_t)width * 4 <= 48 * 1024 && (size_t)s.h * 4 <= 48 * 1024;
  if (dtype == MOE_BF16) return s.h % 64 == 0 && width % 128 == 0;
  return false;
}

size_t ffn_ws_bytes(const moe_shape& s, int32_t width, int32_t dtype) {
  return dtype == MOE_F32 ? ffn_simt_ws_bytes(s) : ffn_tc_ws_bytes(s, width);
}

LayerBufs carve_layer(const moe_shape& s, int32_t act_dtype, void* base) {
  Carver c(base);
  LayerBufs b;
  const size_t Tk = (size_t)s.T * s.k;
  b.logits = c.take<float>((size_t)s.T * s.N);
  b.top_idx = c.take<int32_t>(Tk);
  b.top_w = c.take<float>(Tk);
  b.probs = c.take<float>((size_t)s.T * s.N);
  b.counts = c.take<int32_t>(s.N);
  b.offsets = c.take<int32_t>(s.N + 1);
  b.perm_tok = c.take<int32_t>(Tk);
  b.row_of = c.take<int32_t>(Tk);
  b.overflow = c.take<int32_t>(s.N);
  b.totals = c.take<int32_t>(4);
  b.permute_ws = c.take<char>(std::max(permute_ws_bytes(s),
                                        align_up((size_t)(s.T / 8 + 1) * s.N * 4, 256)));
  b.x_rows = c.take<char>(Tk * s.d * dtype_bytes(act_dtype));
  b.ffn_ws = c.take<char>(ffn_ws_bytes(s, s.d, act_dtype));
  b.y_rows = c.take<float>(Tk * s.d);
  b.row_w = c.take<float>(Tk);
  b.stats_ws = c.take<char>(aux_stats_ws_bytes(s.N));
  b.rd_ws = c.take<char>(route_dispatch_ws_bytes(s));
  b.bytes = c.used();
  return b;
}

// row_w (bf16 only, nullable): store rows row_w[r] * F(u) into y_rows instead
// of F(u).
int run_ffn(const moe_shape& s, int32_t width, const void* x_rows, int32_t dtype,
            const int32_t* offsets, const void* w_gate, const void* w_up, const void* w_down,
            const moe_act& act, float* y_rows, void* ws, cudaStream_t st,
            const float* row_w = nullptr) {
  if (dtype == MOE_F32) {
    return launch_ffn_simt(s, width, static_cast<const float*>(x_rows), offsets,
                           static_cast<const float*>(w_gate), static_cast<const float*>(w_up),
                           static_cast<const float*>(w_down), act, y_rows, ws, st);
  }
  return launch_ffn_tc(s, width, static_cast<const __nv_bfloat16*>(x_rows), offsets,
                       static_cast<const __nv_bfloat16*>(w_gate),
                       static_cast<const __nv_bfloat16*>(w_up),
                       static_cast<const __nv_bfloat16*>(w_down), act, y_rows, ws, st, row_w);
}

bool act_ok(const moe_act* a) {
  if (!a) return false;
  if (a->kind == MOE_ACT_SWIGLU) return true;
  return a->kind == MOE_ACT_SITU_GLU && a->beta_gate > 0.0f && a->beta_up > 0.0f;
}

}  // namespace
}  // namespace moe

extern "C" size_t moe_expert_ffn_workspace_bytes(const moe_shape* shape, int32_t width,
                                                 int32_t dtype) {
  if (!moe::shape_ok(shape) || width <= 0) return 0;
  return moe::ffn_ws_bytes(*shape, width, dtype);
}

extern "C" int moe_expert_ffn(const moe_shape* shape, int32_t width, const void* x_rows,
                              int32_t dtype, const int32_t* offsets, const void* w_gate,
                              const void* w_up, const void* w_down, int32_t w_dtype,
                              const moe_act* act, float* y_rows, void* ws, size_t ws_bytes,
                              void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || width <= 0 || width % 8 != 0 || shape->h <= 0 || !act_ok(act))
    return MOE_ERR_INVALID_ARG;
  if (dtype != w_dtype) return MOE_ERR_UNSUPPORTED;
  if (!ffn_supported(*shape, width, dtype)) return MOE_ERR_UNSUPPORTED;
  if (!offsets || !w_gate || !w_up || !w_down) return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (!x_rows || !y_rows)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_rows) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
      !aligned16(y_rows))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ffn_ws_bytes(*shape, width, dtype) || (!ws && ws_bytes > 0))
    return MOE_ERR_WORKSPACE;
  return run_ffn(*shape, width, x_rows, dtype, offsets, w_gate, w_up, w_down, *act, y_rows, ws,
                 as_stream(stream));
}

extern "C" size_t moe_layer_workspace_bytes(const moe_shape* shape, int32_t act_dtype) {
  if (!moe::shape_ok(shape) || !moe::valid_act_dtype(act_dtype)) return 0;
  return moe::carve_layer(*shape, act_dtype, nullptr).bytes;
}

extern "C" int moe_layer_fwd(const moe_shape* shape, const moe_layer_weights* w, const void* u,
                             int32_t act_dtype, void* y, const moe_layer_outputs* out, void* ws,
                             size_t ws_bytes, void* stream) {
  using namespace moe;
  if (!shape_ok(shape) || !w || !act_ok(&w->act)) return MOE_ERR_INVALID_ARG;
  const moe_shape& s = *shape;
  if (act_dtype != MOE_F32 && act_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (w->w_dtype != act_dtype || !ffn_supported(s, s.d, act_dtype)) return MOE_ERR_UNSUPPORTED;
  if (!w->w_route || !w->w_gate || !w->w_up || !w->w_down) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (!u || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(y) || !aligned16(w->w_route) || !aligned16(w->w_gate) ||
      !aligned16(w->w_up) || !aligned16(w->w_down))
    return MOE_ERR_INVALID_ARG;
  LayerBufs b = carve_layer(s, act_dtype, ws);
  if (!ws || ws_bytes < b.bytes) return MOE_ERR_WORKSPACE;
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
  // bf16 layers: the permutation records each grouped row's combine weight,
  // the down GEMM stores rows a * F(u), and the combine adds them (the down
  // projection carries the multiply of the weighted combine y = sum a F)
  float* row_w = act_dtype == MOE_BF16 ? b.row_w : nullptr;

  int rc;
  if (route_dispatch_ok(s, act_dtype)) {
    // Few experts, token rows fit on chip: routing, permutation and gather in
    // one cooperative launch.
    rc = launch_route_dispatch(s, u, act_dtype, w->w_route, w->bias, top_idx, top_w, probs,
                               nullptr, counts, offsets, perm_tok, row_of, overflow, totals,
                               b.x_rows, b.rd_ws, st, row_w);
    if (rc == MOE_OK && want_stats)
      rc = launch_aux_stats(s.T, s.N, s.k, probs, top_idx, o.f, o.P, o.n_sum_fP, nullptr,
                            b.stats_ws, st);
    if (rc != MOE_OK) return rc;
  } else {
    // Few experts: the router also counts each block's dispatches, and one
    // kernel then scans and scatters (2 launches instead of 4 before the gather).
    const bool small = dispatch_small_ok(s);
    int32_t* hist = small ? static_cast<int32_t*>(b.permute_ws) : nullptr;
    rc = launch_route(s, u, act_dtype, w->w_route, w->bias, top_idx, top_w, probs, b.logits,
                      nullptr, st, hist);
    if (rc != MOE_OK) return rc;
    if (want_stats) {
      rc = launch_aux_stats(s.T, s.N, s.k, probs, top_idx, o.f, o.P, o.n_sum_fP, nullptr,
                            b.stats_ws, st);
      if (rc != MOE_OK) return rc;
    }
    if (small) {
      rc = launch_dispatch_small(s, top_idx, hist, counts, offsets, perm_tok, row_of, overflow,
                                 totals, st, top_w, row_w);
    } else {
      rc = launch_permute(s, top_idx, counts, offsets, perm_tok, row_of, overflow, totals,
                          b.permute_ws, st, top_w, row_w);
    }
    if (rc == MOE_OK) rc = launch_gather(s, s.d, u, act_dtype, perm_tok, offsets, b.x_rows, st);
    if (rc != MOE_OK) return rc;
  }
  rc = run_ffn(s, s.d, b.x_rows, act_dtype, offsets, w->w_gate, w->w_up, w->w_down, w->act,
               b.y_rows, b.ffn_ws, st, row_w);
  if (rc != MOE_OK) return rc;
  if (row_w) return launch_combine_weighted(s, s.d, b.y_rows, row_of, y, act_dtype, st);
  return launch_combine(s, s.d, b.y_rows, row_of, top_w, y, act_dtype, st);
}
