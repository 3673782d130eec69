// Pieces of the backward shared by the layer backward (bwd.cu) and the
// LatentMoE backward (latent_bwd.cu): the routed experts' backward on
// per-expert rows padded to multiples of 64, the router's dz, per-token sums
// of expert-row gradients plus the router term, and the router's weight
// gradient.  Every reduction runs in a fixed order.
#pragma once

#include "common.cuh"

namespace moe {

// Workspace of the experts' backward for `width`-wide expert inputs.
struct BwdBufs {
  int32_t* pad;  // [N+1] padded group offsets
  __nv_bfloat16 *x, *dyr, *dyw, *g, *v, *H, *dG, *dV;
  float *a, *da_part, *dX;
  int64_t rows;  // padded row capacity: T*k + 64 N
  size_t bytes;
};

BwdBufs carve_bwd(const moe_shape& s, int width, void* base);

// The two halves of experts_backward: the forward rows (padded offsets, the
// gathered inputs b.x and weights b.a, the pre-activations b.g, b.v and
// b.H), then the backward rows (the gathered dy, dG, dV, da partials, b.dX
// and the weight gradients).
int experts_forward_rows(const moe_shape& s, int width, const __nv_bfloat16* u,
                         const __nv_bfloat16* Wg, const __nv_bfloat16* Wu, const moe_act& act,
                         const moe_layer_outputs& fwd, const BwdBufs& b, cudaStream_t st);
int experts_backward_rows(const moe_shape& s, int width, const __nv_bfloat16* dy,
                          const __nv_bfloat16* Wg, const __nv_bfloat16* Wu,
                          const __nv_bfloat16* Wd, const moe_act& act,
                          const moe_layer_outputs& fwd, const BwdBufs& b, float* dw_gate,
                          float* dw_up, float* dw_down, cudaStream_t st);

// The grouped experts' backward for inputs u [T][width] and upstream dy
// [T][width] (both bf16), routed as fwd says: recomputes the pre-activations
// and H on the padded rows, then dG, dV and the da partial sums, the input
// gradient rows b.dX [rows][width] fp32 and the weight gradients (fp32,
// gate / up [N][h][width], down [N][width][h]).
int experts_backward(const moe_shape& s, int width, const __nv_bfloat16* u,
                     const __nv_bfloat16* dy, const __nv_bfloat16* Wg, const __nv_bfloat16* Wu,
                     const __nv_bfloat16* Wd, const moe_act& act, const moe_layer_outputs& fwd,
                     const BwdBufs& b, float* dw_gate, float* dw_up, float* dw_down,
                     cudaStream_t st);

// dz [T][N] from the da partial sums of experts_backward, the forward's
// probabilities and weights, and the balancing term (alpha, f nullable).
int bwd_router_dz(const moe_shape& s, const moe_layer_outputs& fwd, const BwdBufs& b, float alpha,
                  const float* f, float* dz, cudaStream_t st);

// out[t] (+)= sum over kept slots of b->dX rows (b nullable: none) + sum_j
// dz[t][j] w_route[j] (w_route nullable: none), out [T][width] fp32.
int bwd_token_sum(const moe_shape& s, int width, const moe_layer_outputs& fwd, const BwdBufs* b,
                  const float* dz, const float* w_route, float* out, bool add, cudaStream_t st);

// dw [N][d] = sum_t dz[t] u[t]^T.
int bwd_router_wgrad(const float* dz, const __nv_bfloat16* u, int T, int N, int d, float* dw,
                     cudaStream_t st);

bool bwd_act_ok(const moe_act& a);

// H = bf16(act(g, v)) over n elements (a multiple of 8), g and v bf16.
int bwd_hidden_rows(const __nv_bfloat16* g, const __nv_bfloat16* v, int64_t n,
                    const moe_act& act, __nv_bfloat16* H, cudaStream_t st);

// tcgen05 backward GEMMs (gemm_bwd.cu); rows: padded row count, offsets: the
// padded group ranges.
int bwd_dgrad_act(const int32_t* offsets, int G, int64_t rows, int width, int h,
                  const __nv_bfloat16* dy_rows, const __nv_bfloat16* w_down,
                  const __nv_bfloat16* g_pre, const __nv_bfloat16* v_pre, const float* row_w,
                  const moe_act& act, __nv_bfloat16* dG, __nv_bfloat16* dV, float* da_part,
                  cudaStream_t st);
int bwd_dgrad_x(const int32_t* offsets, int G, int64_t rows, int width, int h,
                const __nv_bfloat16* dG, const __nv_bfloat16* dV, const __nv_bfloat16* w_gate,
                const __nv_bfloat16* w_up, float* dX, cudaStream_t st);
// out [rows][M] fp32 = B [rows][K] . A, A [G*K][M] read MN-major (one group
// per row range of offsets; K a multiple of 64, M of 128).
int bwd_dgrad_plain(const int32_t* offsets, int G, int64_t rows, int K, int M,
                    const __nv_bfloat16* B, const __nv_bfloat16* A, float* out, cudaStream_t st);
int bwd_wgrad(const int32_t* offsets, int G, int64_t rows, const __nv_bfloat16* A, int M,
              const __nv_bfloat16* B, int Ncols, float* dW, cudaStream_t st);

}  // namespace moe
