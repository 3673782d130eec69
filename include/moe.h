/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts layer forward.
 *
 * The layer (tutorial "Mixture of Experts MoE: how sparse activation saves
 * compute", §3.1-§3.8):
 *   z_t = W_route u_t (+ b)          router logits, fp32          (§3.2 eq. z)
 *   p_t = softmax(z_t)                                             (§3.2 eq. p)
 *   S_t = top-k of z_t, ties to the lower expert index             (§3.2)
 *   a_{t,i} = p_{t,i} / sum_{j in S_t} p_{t,j}   (renorm)          (§3.2 eq. a)
 *   F_i(u) = W_down,i (SiLU(W_gate,i u) * W_up,i u)  SwiGLU expert (§3.1 eq. F)
 *   y_t = sum_{i in S_t, kept} a_{t,i} F_i(u_t)                    (§3.2 eq. y)
 * with tokens grouped by expert and a per-expert capacity C (§3.5, §3.6, §3.8).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers unless a parameter says "host".
 *     The caller owns every buffer; the library never allocates device memory.
 *     Scratch memory is passed as (ws, ws_bytes); its size comes from the
 *     matching *_workspace_bytes query.  Pointers must be 16-byte aligned.
 *   - Row-major layouts.  u [T][d]; W_route [N][d] fp32; bias [N] fp32;
 *     expert weights expert-contiguous: W_gate [N][h][d], W_up [N][h][d],
 *     W_down [N][d][h] (the expert-grouped storage of the deployment notes,
 *     "Kestrel-MCU notes 13", §2).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Host threads: any entry point may be called from several host threads
 *     at once (the lazy per-device setup only repeats idempotent attribute
 *     calls when first calls race).  Two calls whose device work may overlap
 *     must not share a workspace, and moe_permute_noalloc calls must not
 *     overlap at all (one shared scratch).  The device status word is per
 *     device, shared by all streams.
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_*.  Argument errors are
 *     detected on the host, synchronously, before anything is launched.
 *     Errors found by a kernel (an index out of range, a bounded wait that
 *     ran out) are recorded in a sticky device status word that
 *     moe_device_status() reads.  No C++ exception crosses this boundary.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every entry point is exported from the shared library. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* ---------------------------------------------------------------- status */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* null pointer, bad size, misalignment */
#define MOE_ERR_UNSUPPORTED (-2) /* valid but not implemented combination */
#define MOE_ERR_CUDA (-3)        /* a CUDA runtime call failed */
#define MOE_ERR_TIMEOUT (-4)     /* device: a bounded wait ran out */
#define MOE_ERR_BOUNDS (-5)      /* device: an index was out of range */
#define MOE_ERR_WORKSPACE (-6)   /* ws_bytes smaller than the query returned */

/* ------------------------------------------------------------ data types */
#define MOE_F32 0
#define MOE_BF16 1
#define MOE_F16 2
#define MOE_Q4_0 3
#define MOE_E4M3 4 /* OCP FP8 E4M3 codes (1 byte) with one fp32 scale per row */

/* Expert activation.  MOE_ACT_SWIGLU: H = SiLU(g) * v.  MOE_ACT_SITU_GLU:
 * H = SiLU(beta_gate tanh(g / beta_gate)) * beta_up tanh(v / beta_up), the
 * soft-capped gate and up of the Stable LatentMoE demo document (SiTU-GLU),
 * whose product stays below beta_gate * beta_up. */
#define MOE_ACT_SWIGLU 0
#define MOE_ACT_SITU_GLU 1

typedef struct {
  int32_t kind;    /* MOE_ACT_* */
  float beta_gate; /* SiTU-GLU only */
  float beta_up;   /* SiTU-GLU only */
} moe_act;

/* Problem shape.  T tokens of width d, N experts, k experts per token,
 * expert hidden width h.  renorm = 1 uses a = p_S / sum p_S (Mixtral-style
 * top-k, tutorial §3.2); renorm = 0 keeps a = p_S (the Switch top-1
 * multiplier, §3.2 caveat).  capacity = C slots per expert (0 = unlimited);
 * the tutorial's C = ceil(c * dispatches / N) is what moe_capacity computes. */
typedef struct {
  int32_t T;
  int32_t d;
  int32_t N;
  int32_t k;
  int32_t h;
  int32_t renorm;
  int32_t capacity;
} moe_shape;

/* Limits checked on the host: 1 <= k <= min(N, 32); 1 <= N <= 1024;
 * d % 8 == 0; h % 64 == 0 for the bf16 tensor-core experts; T * k < 2^31. */

/* Host-only.  C = ceil(factor * k * T / N), tutorial §3.5 with the top-k
 * dispatch count.  Writes *capacity (host pointer).  factor <= 0 gives 0. */
MOE_API int moe_capacity(int64_t T, int32_t N, int32_t k, double factor, int32_t* capacity);

/* ---------------------------------------------------------------- router */
/* Router, softmax, top-k and combine weights (tutorial §3.2).
 *   u        [T][d] in u_dtype (MOE_F32, MOE_BF16 or MOE_F16)
 *   w_route  [N][d] fp32;  bias [N] fp32 or NULL (added to z after the dot)
 *   top_idx  [T][k] int32 out: experts by descending z, ties to lower index
 *   top_w    [T][k] fp32 out: a (renormalised when shape->renorm)
 *   probs    [T][N] fp32 out or NULL: softmax p
 *   logits   [T][N] fp32 out or NULL: z
 * z is formed in one fixed fp32 order, so routing decisions are reproducible
 * bit for bit: j = 0..d-1 is cut into blocks of 128 (the last may be
 * shorter), each block sum is an ascending fused-multiply-add chain from +0,
 * and z = +0 plus the block sums in ascending order (then + b).
 * Needs ws of moe_route_workspace_bytes(shape) bytes (may be 0 -> ws NULL). */
MOE_API size_t moe_route_workspace_bytes(const moe_shape* shape);
MOE_API int moe_route(const moe_shape* shape, const void* u, int32_t u_dtype, const float* w_route,
              const float* bias, int32_t* top_idx, float* top_w, float* probs, float* logits,
              void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------- aux stats */
/* Switch balancing statistics (tutorial §3.4) from probs [T][N] and top_idx:
 *   f[i] = fraction of tokens whose argmax (slot 0) is i
 *   P[i] = mean over tokens of p[t][i]
 *   n_sum_fP[0] = N * sum_i f[i] P[i]   (L_aux without alpha)
 *   loads[i] = dispatches to expert i over all k slots (L_i, §3.6)
 * Any output may be NULL; probs may be NULL (P and n_sum_fP then read 0).
 * ws: moe_aux_stats_workspace_bytes(N) bytes of scratch. */
MOE_API size_t moe_aux_stats_workspace_bytes(int32_t N);
MOE_API int moe_aux_stats(int32_t T, int32_t N, int32_t k, const float* probs, const int32_t* top_idx,
                  float* f, float* P, float* n_sum_fP, int32_t* loads, void* ws, size_t ws_bytes,
                  void* stream);

/* Gradient of the aux loss with respect to the router logits, with the
 * batch loads held constant (tutorial §3.7):
 *   dz[t][j] = (alpha N / T) p[t][j] (f[j] - sum_i f[i] p[t][i]).
 * probs [T][N] fp32 (moe_route's probs), f [N] fp32 (moe_aux_stats' f),
 * dz [T][N] fp32 out.  fp32 arithmetic (max|error| about 1e-6 of max|dz|).
 * T = 0 is a no-op. */
MOE_API int moe_aux_grad(int32_t T, int32_t N, float alpha, const float* probs, const float* f,
                         float* dz, void* stream);

/* --------------------------------------------------------------- permute */
/* Group the T*k dispatches by expert (tutorial §3.5, §3.6, §3.8).
 * Dispatch (t, s) -> expert top_idx[t][s]; its rank = dispatches to the same
 * expert from lower tokens; kept iff capacity == 0 or rank < capacity.
 *   counts   [N]   L_e, all dispatches
 *   offsets  [N+1] exclusive prefix sum of the kept counts; offsets[N] = rows
 *   perm_tok [T*k] token of grouped row r, for r < offsets[N]
 *   row_of   [T][k] grouped row of (t, s), or -1 when dropped
 *   overflow [N]   max(L_e - C, 0)
 *   totals   [3]   {kept rows, overflowed dispatches, empty slots sum max(C - L_e, 0)}
 * Bit-exact and deterministic.  ws: moe_permute_workspace_bytes(shape). */
MOE_API size_t moe_permute_workspace_bytes(const moe_shape* shape);
MOE_API int moe_permute(const moe_shape* shape, const int32_t* top_idx, int32_t* counts,
                int32_t* offsets, int32_t* perm_tok, int32_t* row_of, int32_t* overflow,
                int32_t* totals, void* ws, size_t ws_bytes, void* stream);

/* Allocation-free moe_permute.  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory when they call
 * in (a C program that loads only this library and has no device allocator,
 * or a framework whose memory planner forbids allocation at call time).
 * Same arguments, results and errors as moe_permute, minus (ws, ws_bytes):
 * the scratch is a fixed 1 MiB array inside the library, resident on every
 * GPU that loads it until the process exits.  Limit: ceil(T*k / 256) * N
 * <= 262144 (e.g. T*k = 65536 dispatches with N up to 1024 experts); larger
 * problems return MOE_ERR_WORKSPACE before anything is launched.  The first
 * call on a device looks up the array's device address (with that device
 * current); make that first call before any stream capture.  All calls in
 * the process share the one array, so calls whose work overlaps on the GPU
 * (other streams, other host threads) race; serialise them.  Nothing in the
 * array needs to start at zero: each call rewrites what it reads.  Never
 * calls cudaMalloc, cudaFree or any allocating routine. */
MOE_API int moe_permute_noalloc(const moe_shape* shape, const int32_t* top_idx, int32_t* counts,
                                int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                                int32_t* overflow, int32_t* totals, void* stream);

/* ---------------------------------------------------------------- gather */
/* x_rows[r] = u[perm_tok[r]] for r < offsets[N] (tutorial §3.6: expert i
 * receives its [L_i, d] rows).  u [T][width] in dtype; x_rows has room for
 * T*k rows of width elements.  Rows >= offsets[N] are left untouched.  An
 * offsets[N] outside [0, T*k] or a perm_tok entry outside [0, T) records
 * MOE_ERR_BOUNDS in the device status word; no row beyond T*k is written
 * and a row with a bad token id is skipped. */
MOE_API int moe_gather(const moe_shape* shape, int32_t width, const void* u, int32_t dtype,
               const int32_t* perm_tok, const int32_t* offsets, void* x_rows, void* stream);

/* ------------------------------------------------------------ expert FFN */
/* Grouped expert FFN on grouped rows (tutorial §3.1): for every grouped row
 * r of expert e (offsets[e] <= r < offsets[e+1]):
 *   y_rows[r] = W_down,e act(W_gate,e x_rows[r], W_up,e x_rows[r])
 * unweighted, fp32 [T*k][width].  width is the expert input/output width (d,
 * or the latent width of a latent-space layer); h = shape->h.
 * dtype = w_dtype = MOE_F32 (SIMT fp32) or MOE_BF16 (tcgen05 tensor cores,
 * fp32 accumulate, hidden stored as bf16).  ws: moe_expert_ffn_workspace_bytes. */
MOE_API size_t moe_expert_ffn_workspace_bytes(const moe_shape* shape, int32_t width, int32_t dtype);
MOE_API int moe_expert_ffn(const moe_shape* shape, int32_t width, const void* x_rows, int32_t dtype,
                   const int32_t* offsets, const void* w_gate, const void* w_up,
                   const void* w_down, int32_t w_dtype, const moe_act* act, float* y_rows,
                   void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------- combine */
/* y[t] = sum over kept slots s (row_of[t][s] >= 0, ascending s) of
 * top_w[t][s] * y_rows[row_of[t][s]]  (tutorial §3.2 eq. y); dropped slots
 * add nothing and the weights are not renormalised.  y [T][width] in y_dtype
 * (MOE_F32, MOE_BF16 or MOE_F16), fully overwritten.  A row_of entry at or
 * above T*k (y_rows holds T*k rows) records MOE_ERR_BOUNDS in the device
 * status word and that slot adds nothing. */
MOE_API int moe_combine(const moe_shape* shape, int32_t width, const float* y_rows,
                const int32_t* row_of, const float* top_w, void* y, int32_t y_dtype,
                void* stream);

/* ------------------------------------------------------------ full layer */
typedef struct {
  const float* w_route; /* [N][d] fp32 */
  const float* bias;    /* [N] fp32 or NULL */
  const void* w_gate;   /* [N][h][d] */
  const void* w_up;     /* [N][h][d] */
  const void* w_down;   /* [N][d][h] */
  int32_t w_dtype;      /* MOE_F32 or MOE_BF16 (same as the activations) */
  moe_act act;
} moe_layer_weights;

/* Optional device outputs of moe_layer_fwd; every pointer may be NULL. */
typedef struct {
  int32_t* top_idx;  /* [T][k] */
  float* top_w;      /* [T][k] */
  float* probs;      /* [T][N] */
  int32_t* counts;   /* [N] */
  int32_t* offsets;  /* [N+1] */
  int32_t* perm_tok; /* [T*k] */
  int32_t* row_of;   /* [T][k] */
  int32_t* overflow; /* [N] */
  int32_t* totals;   /* [3] */
  float* f;          /* [N] */
  float* P;          /* [N] */
  float* n_sum_fP;   /* [1] */
} moe_layer_outputs;

/* The whole forward: router -> permute -> gather -> grouped SwiGLU experts ->
 * weighted combine, plus the aux statistics when out->f/P/n_sum_fP are set.
 * u and y are [T][d] in act_dtype (MOE_F32 or MOE_BF16).  y excludes the
 * residual: a dropped dispatch contributes zero (tutorial §3.5: the
 * residual path carries it).  ws: moe_layer_workspace_bytes.  For few
 * experts whose token rows fit on chip, routing, permutation and gather run
 * as one cooperative launch whose grid-barrier words live in ws (zeroed by
 * the call), so a workspace serves one call at a time; results are the same
 * bit for bit on either path.  Capturable in a CUDA graph. */
MOE_API size_t moe_layer_workspace_bytes(const moe_shape* shape, int32_t act_dtype);
MOE_API int moe_layer_fwd(const moe_shape* shape, const moe_layer_weights* w, const void* u,
                  int32_t act_dtype, void* y, const moe_layer_outputs* out, void* ws,
                  size_t ws_bytes, void* stream);

/* ---------------------------------------------------------- layer backward */
/* Gradients of L = sum_t dy_t . y_t + alpha N sum_i f_i P_i for the bf16 layer
 * of moe_layer_fwd (tutorial §3.1, §3.2; §3.4 P_i = mean_t p_ti; §3.7 the
 * balancing term's gradient with the loads f held fixed), with the forward's
 * selected sets and capacity drops held fixed (top-k and the capacity cut
 * are piecewise constant): a dropped dispatch gets no gradient, and only the
 * selected experts of kept dispatches get weight gradient.
 *   dz [T][N]         dL/dz (router logits): renormalisation and softmax
 *                     backward of da_s = dy_t . F_{e_s}(u_t), plus the term
 *                     (alpha N / T) p_tj (f_j - sum_i f_i p_ti) when f != NULL
 *   du [T][d]         dL/du: the experts' input gradients of the kept slots
 *                     plus sum_j dz_tj W_route[j]
 *   dw_route [N][d]   sum_t dz_t u_t^T (nullable: not formed)
 *   dw_gate, dw_up [N][h][d], dw_down [N][d][h]   every expert's matrix,
 *                     zero for an expert with no kept dispatch
 * All fp32, device, caller-owned, fully overwritten. */
typedef struct {
  float* du;
  float* dz;
  float* dw_route;
  float* dw_gate;
  float* dw_up;
  float* dw_down;
} moe_layer_grads;

MOE_API size_t moe_layer_bwd_workspace_bytes(const moe_shape* shape);
/* shape, w, u as for moe_layer_fwd (bf16 experts; h and d multiples of 128);
 * dy [T][d] bf16; fwd: the forward's top_idx, top_w, probs, offsets,
 * perm_tok and row_of (moe_layer_fwd fills them when they are requested in
 * its outputs).  The expert GEMMs run on the tensor cores (bf16 operands,
 * fp32 accumulate, the weights and token rows read in their stored layout);
 * every reduction has a fixed order, so the result is reproducible.
 * Returns MOE_ERR_INVALID_ARG for NULL or misaligned pointers or unsupported
 * widths, MOE_ERR_UNSUPPORTED for non-bf16 experts, MOE_ERR_WORKSPACE for a
 * short workspace. */
MOE_API int moe_layer_bwd(const moe_shape* shape, const moe_layer_weights* w, const void* u,
                          const void* dy, const moe_layer_outputs* fwd, float alpha,
                          const float* f, const moe_layer_grads* grads, void* ws,
                          size_t ws_bytes, void* stream);

/* -------------------------------------------------------------- LatentMoE */
/* Latent-space MoE layer (Stable LatentMoE demo document: width separation,
 * RMSNorm before the up-projection, SiTU-GLU soft caps).  The routed experts
 * work in a latent width l < d, the shared experts at full width d:
 *   z = W_route x (+b) on the full-width x; top-k; a   (routing on x)
 *   x_l = W_dp x                                 W_dp [l][d] bf16
 *   m = sum_s a_s E_{e_s}(x_l)                   routed gate/up [N][h][l], down [N][l][h]
 *   m^ = m / sqrt(mean(m^2) + rms_eps)           no gain
 *   y = W_upp m^ + sum_j S_j(x)                  W_upp [d][l]; S_j SwiGLU d -> sh -> d
 * The routed act is taken from moe_layer_weights.act (MOE_ACT_SITU_GLU with
 * beta_gate, beta_up for the document's experts); shared experts are plain
 * SwiGLU.  Capacity applies as in moe_layer_fwd. */
typedef struct {
  int32_t latent;          /* l, multiple of 128 */
  int32_t n_shared;        /* 0..2 shared experts */
  int32_t shared_hidden;   /* sh, multiple of 64 */
  const void* w_down_proj; /* [l][d] bf16 */
  const void* w_up_proj;   /* [d][l] bf16 */
  const void* shared_gate; /* [n_shared][sh][d] bf16 */
  const void* shared_up;   /* [n_shared][sh][d] bf16 */
  const void* shared_down; /* [n_shared][d][sh] bf16 */
  float rms_eps;
} moe_latent_weights;

MOE_API size_t moe_latent_workspace_bytes(const moe_shape* shape, const moe_latent_weights* lw);
/* shape: T tokens, d model width, N routed experts, k, h routed hidden width.
 * w: router [N][d] fp32 (+bias) and the routed experts (bf16, latent width),
 * w->w_dtype == MOE_BF16.  x, y [T][d] bf16.  out: as for moe_layer_fwd.
 * Returns MOE_ERR_INVALID_ARG for unsupported widths, NULL or misaligned
 * pointers or non-positive SiTU-GLU caps, MOE_ERR_UNSUPPORTED for non-bf16
 * experts, MOE_ERR_WORKSPACE for a short workspace. */
MOE_API int moe_latent_fwd(const moe_shape* shape, const moe_layer_weights* w,
                           const moe_latent_weights* lw, const void* x, void* y,
                           const moe_layer_outputs* out, void* ws, size_t ws_bytes, void* stream);

/* FP8 routed experts (Stable LatentMoE demo document, SiTU-GLU: the soft caps
 * bound the hidden product by beta_g * beta_u = 100, under E4M3's largest
 * finite value 448, which is what FP8 experts need).  Values are
 * scale[row] * e4m3(code[row][col]) (OCP E4M3: bias 7, no infinity, 448 the
 * largest finite value); moe_quantize_e4m3_rows makes them from bf16 or fp32
 * rows: s = amax(row) / 448 (1 for a zero row), code = e4m3(x / s) rounded to
 * nearest even and saturated at 448, each division one fp32 operation. */
typedef struct {
  const float* gate_scale; /* [N * h] row scales of w_gate's codes */
  const float* up_scale;   /* [N * h] row scales of w_up's codes */
  const float* down_scale; /* [N * l] row scales of w_down's codes */
} moe_e4m3_scales;

/* x: [rows][cols] in x_dtype (MOE_BF16 or MOE_F32), cols a multiple of 16;
 * codes [rows][cols] bytes and scales [rows] fp32 (device, caller-owned).
 * Asynchronous on stream.  MOE_ERR_INVALID_ARG for a bad size, NULL or
 * misaligned pointer (x and codes 16-B aligned, scales 4-B aligned),
 * MOE_ERR_UNSUPPORTED for another x_dtype. */
MOE_API int moe_quantize_e4m3_rows(int64_t rows, int32_t cols, const void* x, int32_t x_dtype,
                                   uint8_t* codes, float* scales, void* stream);

/* The grouped expert FFN of moe_expert_ffn with E4M3 operands: x_rows
 * [T*k][width] codes with x_scale [T*k] (one scale per row, e.g. from
 * moe_quantize_e4m3_rows), the experts' E4M3 codes (gate, up [N][h][width],
 * down [N][width][h]) with their row scales, SiTU-GLU or SwiGLU; H is stored
 * as E4M3 codes with no scale in ws; y_rows [T*k][width] fp32, F(u) of each
 * grouped row (not weighted).  width and h multiples of 128.
 * ws: moe_expert_ffn_e4m3_workspace_bytes.  Errors as moe_expert_ffn. */
MOE_API size_t moe_expert_ffn_e4m3_workspace_bytes(const moe_shape* shape);
MOE_API int moe_expert_ffn_e4m3(const moe_shape* shape, int32_t width, const uint8_t* x_rows,
                                const float* x_scale, const int32_t* offsets,
                                const uint8_t* w_gate, const uint8_t* w_up,
                                const uint8_t* w_down, const moe_e4m3_scales* scales,
                                const moe_act* act, float* y_rows, void* ws, size_t ws_bytes,
                                void* stream);

/* The LatentMoE layer of moe_latent_fwd with E4M3 routed experts: w->w_dtype
 * == MOE_E4M3 and w->w_gate, w_up, w_down hold codes (gate, up [N][h][l],
 * down [N][l][h] bytes) with the row scales in *scales.  x_l = W_dp x (bf16)
 * is quantised per token the same way as the weights; the gate/up and down
 * GEMMs run on the FP8 tensor cores (E4M3 x E4M3, fp32 accumulate) with the
 * scales applied to the fp32 results; H is stored as E4M3 codes with no
 * scale.  The router, W_dp, W_upp and the shared experts stay bf16 / fp32.
 * Requires l and h multiples of 128.  Workspace: moe_latent_workspace_bytes.
 * Errors as moe_latent_fwd; MOE_ERR_INVALID_ARG when scales or one of its
 * pointers is NULL. */
MOE_API int moe_latent_fwd_e4m3(const moe_shape* shape, const moe_layer_weights* w,
                                const moe_e4m3_scales* scales, const moe_latent_weights* lw,
                                const void* x, void* y, const moe_layer_outputs* out, void* ws,
                                size_t ws_bytes, void* stream);

/* Gradients of L = sum_t dy_t . y_t for the LatentMoE layer of
 * moe_latent_fwd (bf16 routed experts), with the forward's selected sets held
 * fixed (the reading of the layer backward above): through y = W_upp m^ +
 * sum_j S_j(x), the RMSNorm m^ = m / sqrt(mean(m^2) + eps), the routed
 * experts on x_l = W_dp x and the router on x.  All fp32, device,
 * caller-owned, fully overwritten:
 *   dx [T][d], dz [T][N], dw_route [N][d] (nullable), dw_gate, dw_up
 *   [N][h][l], dw_down [N][l][h], dw_dp [l][d], dw_upp [d][l], dsh_gate,
 *   dsh_up [n_shared][sh][d], dsh_down [n_shared][d][sh] (with shared
 *   experts). */
typedef struct {
  float* dx;
  float* dz;
  float* dw_route;
  float* dw_gate;
  float* dw_up;
  float* dw_down;
  float* dw_dp;
  float* dw_upp;
  float* dsh_gate;
  float* dsh_up;
  float* dsh_down;
} moe_latent_grads;

MOE_API size_t moe_latent_bwd_workspace_bytes(const moe_shape* shape,
                                              const moe_latent_weights* lw);
/* w, lw, x as for moe_latent_fwd (d, l, h and sh multiples of 128); dy
 * [T][d] bf16; fwd: that forward's top_idx, top_w, probs, offsets, perm_tok
 * and row_of.  The GEMMs run on the tensor cores (bf16 operands, fp32
 * accumulate); every reduction has a fixed order.  Errors as
 * moe_layer_bwd. */
MOE_API int moe_latent_bwd(const moe_shape* shape, const moe_layer_weights* w,
                           const moe_latent_weights* lw, const void* x, const void* dy,
                           const moe_layer_outputs* fwd, const moe_latent_grads* grads, void* ws,
                           size_t ws_bytes, void* stream);

/* ---------------------------------------------------------- q4_0 decode */
/* Small-batch decode with q4_0 experts (deployment notes "Kestrel-MCU notes
 * 13", §2 lookup loading of the selected experts only, §4 q4_0 experts with an
 * fp32 router).  q4_0: blocks of 32 consecutive values along a row, one fp16
 * scale s per block, 4-bit q in 0..15, w = (q - 8) s; byte j of a block holds
 * element j (low nibble) and element j + 16 (high nibble).  A matrix
 * [rows][cols] is qs [rows][cols/2] bytes plus scales [rows][cols/32] fp16.
 * Per layer: gate, up [N][h][d]; down [N][d][h]; router [N][d] fp32. */
typedef struct {
  const float* w_route;        /* [N][d] fp32 */
  const float* bias;           /* [N] fp32 or NULL */
  const uint8_t* gate_qs;      /* [N][h][d/2] */
  const uint16_t* gate_scales; /* [N][h][d/32] fp16 */
  const uint8_t* up_qs;
  const uint16_t* up_scales;
  const uint8_t* down_qs;      /* [N][d][h/2] */
  const uint16_t* down_scales; /* [N][d][h/32] fp16 */
} moe_q4_layer;

/* Limits: T <= 32, N <= 64, k <= 8, d % 32 == 0, h % 32 == 0, h / 32 a
 * divisor of 32, and the kernel's per-CTA shared-memory plan (token rows,
 * router rows, one phase-A item, the selected experts' down rows of one
 * output slice) within 226 KB.  Returns 0 for shapes outside them.  The
 * workspace holds the hidden vectors, the routing scratch, the chained
 * activations and the grid-barrier words; one call at a time per workspace.
 * The two decode calls return MOE_ERR_INVALID_ARG for a shape outside these
 * limits, a NULL or misaligned weight or activation pointer (q4 planes and
 * the router 16-byte aligned, scales and bias 4-byte aligned),
 * MOE_ERR_WORKSPACE for a short workspace, and MOE_OK at once for T = 0. */
MOE_API size_t moe_decode_workspace_bytes(const moe_shape* shape);

/* One decode layer: u [T][d] fp16 (bit patterns) -> y [T][d] fp16, the
 * layer output sum_s a_s F_{e_s}(u_t) with the hidden vector kept in fp32;
 * u_next (nullable) = fp16(u + y), the next layer's input.  top_idx [T][k]
 * and top_w [T][k] are optional outputs.  Only the experts some token
 * selected are read.  `layer` is a host struct of device pointers. */
MOE_API int moe_decode_layer(const moe_shape* shape, const moe_q4_layer* layer, const uint16_t* u,
                             uint16_t* y, uint16_t* u_next, int32_t* top_idx, float* top_w,
                             void* ws, size_t ws_bytes, void* stream);

/* Which kernel moe_decode_layer and moe_decode_step run for this shape on
 * the current device: 1 the per-token kernel, 2 the two-phase kernel, 0 the
 * shape is outside the limits above (or no device is visible). */
MOE_API int moe_decode_kernel(const moe_shape* shape);

/* n_layers chained layers: u_{l+1} = fp16(u_l + y_l), u_out = u_{n_layers}.
 * `layers` is a host array of n_layers structs.  top_idx_all [n_layers][T][k]
 * (nullable) receives every layer's routing.  Up to 32 layers run in one
 * launch (at most one CTA per SM; the two-phase kernel is a cooperative
 * launch whose grid-barrier waits are bounded: MOE_ERR_TIMEOUT in the device
 * status word).  When the T k (token, slot)
 * pairs fit one CTA each, its shared-memory plan fits and a cluster of a
 * token's CTAs can be resident, the launch runs
 * the per-token kernel (CTA = (token, slot, hidden slice) for all layers,
 * the token's k S CTAs one thread-block cluster that exchanges partial
 * output rows through distributed shared memory, no grid barrier);
 * otherwise a two-phase kernel (selected-expert
 * hidden slices, grid barrier, (token, output rows) units, grid barrier).
 * The kernel is chosen from the shape, so a chain and moe_decode_layer use
 * the same per-layer arithmetic and a chain equals the layer calls made one
 * by one.  Capturable in a CUDA graph. */
MOE_API int moe_decode_step(const moe_shape* shape, int32_t n_layers, const moe_q4_layer* layers,
                            const uint16_t* u0, uint16_t* u_out, int32_t* top_idx_all, void* ws,
                            size_t ws_bytes, void* stream);

/* moe_decode_step that also records, for each layer, 13 SM-cycle stamps
 * (clock64 of block 0, thread 0) into stamps [n_layers][13] (device memory,
 * 8-byte aligned; caller-owned).  Per-token kernel (block 0 = token 0,
 * slot 0, slice 0): 0 layer start, 1 = 0, 2 routed, 3 = 2, 4 the slice's
 * gate/up rows staged, 5 = 4, 6 gate/up dots formed, 7 H formed, 8 = 7,
 * 9 down columns ready, 10 partial output row in shared memory, 11 the
 * cluster barrier passed (every partial row of the token stored), 12 next
 * row formed.
 * Two-phase kernel: 0 layer start, 1 input rows staged, 2 routed, 3
 * dispatch pairs grouped by expert, 4 gate/up q4 rows staged, 5 = 4, 6
 * gate/up dots formed, 7 hidden phase done (H stored), 8 first grid barrier
 * passed, 9 down rows ready, 10 down dots formed, 11 output phase done
 * (u_next stored), 12 second grid barrier passed.  Stamps 4-11 time block
 * 0's first item (equal to the stamp after them when it has none).
 * Differences are cycles of that SM's clock; results are identical to
 * moe_decode_step.
 * MOE_ERR_INVALID_ARG for a null or misaligned stamps pointer. */
MOE_API int moe_decode_step_trace(const moe_shape* shape, int32_t n_layers,
                                  const moe_q4_layer* layers, const uint16_t* u0, uint16_t* u_out,
                                  int32_t* top_idx_all, void* ws, size_t ws_bytes,
                                  uint64_t* stamps, void* stream);

/* ---------------------------------------------------- quantile balancing */
/* Quantile balancing of the expert biases ("Stable LatentMoE interactive demo
 * document", Quantile Balancing).  scores [T][N] fp32 are the router logits,
 * bias [N] fp32 (nullable = 0) the current balancing bias.  With every
 * token's cutoff a_i = the k-th largest s_ij + b_j held fixed, expert j takes
 * token i iff b_j >= required_ij = a_i - s_ij, so the bias giving expert j q
 * tokens is the q-th smallest required_ij:
 *   cutoff [T]      (nullable: kept in the workspace) a_i;
 *   bias_exact [N]  the q-th smallest required_ij (a zero as +0);
 *   bias_hist [N]   (nullable, needs bins >= 1) the histogram estimate: bins
 *                   equal bins over the [min, max] of required_j, the upper
 *                   edge of the first bin whose running count reaches q;
 *   loads [N]       (nullable) #{i : required_ij <= bias_exact_j} (q, or more
 *                   through ties).
 * Every step is one fp32 operation in a fixed order (bit-reproducible).
 * Limits: 1 <= T <= 32768, 1 <= N <= 1024, 1 <= k <= min(N, 32),
 * 1 <= q <= T, 0 <= bins <= 4096.  Device pointers, caller-owned.
 * Returns MOE_ERR_INVALID_ARG outside the limits or for NULL scores or
 * bias_exact, MOE_ERR_WORKSPACE when cutoff is NULL and ws is shorter than
 * moe_quantile_balance_workspace_bytes(T, N). */
MOE_API size_t moe_quantile_balance_workspace_bytes(int32_t T, int32_t N);
MOE_API int moe_quantile_balance(int32_t T, int32_t N, int32_t k, const float* scores,
                                 const float* bias, int32_t q, int32_t bins, float* cutoff,
                                 float* bias_exact, float* bias_hist, int32_t* loads, void* ws,
                                 size_t ws_bytes, void* stream);

/* -------------------------------------------------- expert parallelism */
/* Exchange plan of expert parallelism, host only (no device work).  world
 * ranks, N experts, expert e held by rank e / (N / world).  An expert's
 * capacity counts the dispatches of all ranks in one global order (rank 0's
 * tokens first, then rank 1's, each in token order), so the expert-parallel
 * layer equals the single-device layer (tutorial §3.5, §3.6, §3.8) on the
 * ranks' batches laid end to end.  Input, host:
 *   counts_all [world][N]  every rank's dispatches per expert, before capacity
 *                          (each rank's moe_permute counts with capacity 0)
 * Outputs for `rank`, host, all overwritten (E = N / world):
 *   kept [N]            my dispatches to e that fit: the first kept[e] of my
 *                       run of dispatches to e in token order
 *   local_offsets [N+1] my grouped layout of kept rows (exclusive prefix)
 *   send_base [N]       row of the owner's receive buffer where my kept rows
 *                       for e start; my j-th kept dispatch to e lands there + j
 *   send_counts [world] rows I send to each rank (its experts, in order)
 *   recv_offsets [E+1]  my receive buffer grouped by my local experts, then by
 *                       source rank, then by the source's token order
 *   recv_src_base [E][world]  row where source r's rows for local expert el
 *                       start (results go back from there)
 *   recv_counts [world] rows I receive from each rank
 *   overflow [N]        (nullable) dropped dispatches of all ranks per expert
 * Returns MOE_ERR_INVALID_ARG when N % world != 0, rank or capacity is out
 * of range, a count is negative, a pointer is NULL, or a row count exceeds
 * 2^31 - 1. */
MOE_API int moe_ep_plan(int32_t world, int32_t rank, int32_t N, int32_t capacity,
                        const int32_t* counts_all, int32_t* kept, int32_t* local_offsets,
                        int32_t* send_base, int32_t* send_counts, int32_t* recv_offsets,
                        int32_t* recv_src_base, int32_t* recv_counts, int32_t* overflow);

/* Expert parallelism, device side: the dispatch and combine all-to-alls the
 * tutorial names as the multi-device cost of experts split over devices,
 * each fused with its neighbouring step (the gather, the weighted combine).
 * Rank r owns experts [r E, (r+1) E), E = N / world.  Every rank holds, in
 * its own device memory, the buffers below; the peer_* arrays (device
 * memory, [world] entries) hold every rank's buffers as addresses this
 * device can load and store (peer memory over NVLink after
 * cudaDeviceEnablePeerAccess or an IPC / symmetric-memory mapping; plain
 * device addresses when the ranks share one device).  No TMA and no
 * multicast touch peer memory: plain loads and stores only. */
typedef struct {
  int32_t world, rank;
  int32_t recv_capacity;       /* rows of recv_rows / out_rows on every rank */
  void* recv_rows;             /* this rank: received token rows, bf16 [recv_capacity][d] */
  float* recv_w;               /* this rank: their combine weights [recv_capacity] */
  void* out_rows;              /* this rank: weighted expert outputs a * F(u), fp32 [recv_capacity][d] */
  uint32_t* arrive;            /* this rank: arrival flags [world], one per source */
  uint32_t* done;              /* this rank: one flag, experts finished */
  void* const* peer_recv_rows; /* [world] every rank's recv_rows */
  float* const* peer_recv_w;   /* [world] every rank's recv_w */
  void* const* peer_out_rows;  /* [world] every rank's out_rows */
  uint32_t* const* peer_arrive;/* [world] every rank's arrive */
  uint32_t* const* peer_done;  /* [world] every rank's done */
} moe_ep_buffers;

/* One step, per rank, on its stream, in this order (epoch = the step number,
 * starting at 1; flags are never reset, a later epoch supersedes):
 *   moe_route, moe_permute with capacity 0 (counts, offsets, perm_tok, row_of
 *   of this rank's dispatches), an all-gather of the counts (NCCL), then
 *   moe_ep_plan on the host and a copy of kept / send_base to the device;
 *   moe_ep_dispatch: every kept dispatch's row of u (bf16 [T][d]) and its
 *     combine weight top_w are stored into the owner's recv buffers at the
 *     plan's row; the last CTA raises arrive[rank] on every rank (release,
 *     system scope) -- also when this rank sends nothing;
 *   moe_ep_expert_ffn: waits until every source's arrival flag reached epoch,
 *     runs this rank's E experts (moe_expert_ffn's kernels; expert_shape:
 *     T = recv_capacity, k = 1, N = E, d, h) on the received rows grouped by
 *     recv_offsets [E+1] (the plan's), stores fp32 rows a * F(u) into
 *     out_rows and raises done;
 *   moe_ep_combine: waits until every rank's done flag reached epoch, then
 *     y_t = sum over kept slots (ascending s) of the owners' out_rows rows,
 *     loaded from their memory; y bf16 [T][d], fully overwritten.
 * With the plan's global order (rank 0's rows of an expert first), y equals
 * the single-device layer on the ranks' batches laid end to end.  A rank
 * reuses its buffers next step only after its own combine, which follows
 * every owner's done flag, so the flags order every overwrite.  Every wait
 * is bounded (about 2 s) and records MOE_ERR_TIMEOUT in the status word; a
 * destination row beyond recv_capacity records MOE_ERR_BOUNDS and is not
 * stored.  ws: moe_ep_workspace_bytes(expert_shape), separate per rank. */
MOE_API size_t moe_ep_workspace_bytes(const moe_shape* expert_shape);
MOE_API int moe_ep_dispatch(const moe_shape* shape, const moe_ep_buffers* bufs, uint32_t epoch,
                            const void* u, const int32_t* perm_tok, const int32_t* offsets,
                            const int32_t* row_of, const float* top_w, const int32_t* kept,
                            const int32_t* send_base, void* ws, size_t ws_bytes, void* stream);
MOE_API int moe_ep_expert_ffn(const moe_shape* expert_shape, const moe_ep_buffers* bufs,
                              uint32_t epoch, const int32_t* recv_offsets, const void* w_gate,
                              const void* w_up, const void* w_down, const moe_act* act, void* ws,
                              size_t ws_bytes, void* stream);
MOE_API int moe_ep_combine(const moe_shape* shape, const moe_ep_buffers* bufs, uint32_t epoch,
                           const int32_t* top_idx, const int32_t* row_of, const int32_t* offsets,
                           const int32_t* kept, const int32_t* send_base, void* y, void* stream);

/* ----------------------------------------------------------- diagnostics */
/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(int32_t status);
/* Synchronises `stream`, then copies the sticky device status word to
 * *status (host pointer): MOE_OK or the first MOE_ERR_* a kernel recorded. */
MOE_API int moe_device_status(void* stream, int32_t* status);
/* Clears the device status word (asynchronous on stream). */
MOE_API int moe_reset_device_status(void* stream);

/* Failure-detection check of the bounded device waits (no counterpart on the
 * pages; it tests this library's own error path).  Launches one small kernel
 * that runs the named wait on a condition nothing satisfies:
 *   MOE_WAIT_GRID_BARRIER  the grid barrier of the cooperative kernels (two
 *                          co-resident CTAs wait for one arrival too many),
 *   MOE_WAIT_MBARRIER      the mbarrier wait of the tcgen05 kernels (a fresh
 *                          barrier whose first phase never completes).
 * The wait gives up after about budget_ns nanoseconds (1e3 .. 2e9), records
 * MOE_ERR_TIMEOUT in the status word and the kernel returns, so the context
 * stays usable: moe_device_status then reads MOE_ERR_TIMEOUT until
 * moe_reset_device_status.  Asynchronous on stream.  Returns
 * MOE_ERR_INVALID_ARG for an unknown kind or a budget out of range.  The
 * grid-barrier check keeps its counter in a fixed device array shared by
 * all calls, so calls that overlap on the GPU race. */
#define MOE_WAIT_GRID_BARRIER 0
#define MOE_WAIT_MBARRIER 1
MOE_API int moe_wait_check(int32_t kind, int64_t budget_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
