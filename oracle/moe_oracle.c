/*
 * CPU oracle for the sparse Mixture-of-Experts SwiGLU layer forward and its
 * backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The GPU product path
 * never links, imports or calls it, and it shares no code with the GPU path.
 *
 * Sources, cited by page title and section:
 *   [MoE tutorial]  "Mixture of Experts MoE: how sparse activation saves
 *                   compute" (jefxiong.cn), §3.1-§3.8 and its appendix lab.
 *   [MCU #13]       "Kestrel-MCU notes 13: the deployment gap between the
 *                   converter and the inference kernel" (0539edu.com), §2, §4, §6.
 *   [MCU #10]       "Kestrel-MCU notes 10: MoE sparsification in practice"
 *                   (gsyq.cn), §3 (bandwidth gain table).
 *   [LatentMoE]     "Stable LatentMoE interactive demo document" (cnblogs via
 *                   82so.com): width separation, RMSNorm before up-projection,
 *                   SiTU-GLU soft caps.
 *
 * Precision: every floating-point quantity is evaluated in double from the
 * exact input values, except the router logits.  The tutorial's router works
 * in fp32 (§3.2 and its code: softmax of logits.float()); the logits decide
 * the discrete top-k, so they are formed in fp32 in one fixed summation order
 * (or_router_logit below) which any implementation can reproduce bit for bit.
 * The layer backward at the end of the file forms the logits in double too:
 * it is the exact-arithmetic gradient, not a replay of the routing decision.
 * Compiled with -ffp-contract=off so each operation rounds on its own.
 *
 * Parity pins: every function is checked against worked numbers printed on
 * the pages, closed forms, brute force or textbook identities in
 * tests/test_oracle_pins.py, tests/test_oracle_backward.py (the backward) and
 * tests/test_oracle_fp8.py (the E4M3 pieces).  The softmax/SiLU/tanh
 * transcendental values themselves have no printed example beyond the
 * tutorial's aux-loss figures.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the oracle's parallel loops use (for reporting its timings), and a
 * way to change them; 1 without OpenMP. */
int or_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void or_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------ formats */

/* bf16 bit pattern -> exact double (the upper half of an IEEE binary32). */
double or_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* IEEE binary16 bit pattern -> exact double, decoded field by field.
 * Subnormals are mantissa * 2^-24 (exponent field 0 means 2^(1-15) with no
 * implicit bit).  [MCU #13] §6 reports a hand-written decoder whose subnormal
 * branch was off by one in the exponent and halved 14.2% of the q4 scales. */
double or_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int ex = (h >> 10) & 0x1F;
  int man = h & 0x3FF;
  double v;
  if (ex == 0) {
    v = ldexp((double)man, -24);
  } else if (ex == 31) {
    v = man ? NAN : INFINITY;
  } else {
    v = ldexp((double)(man | 0x400), ex - 25);
  }
  return sign ? -v : v;
}

/* Storage of an activation or weight tensor. */
enum { OR_F32 = 0, OR_BF16 = 1, OR_F16 = 2, OR_Q4_0 = 3, OR_F64 = 4, OR_E4M3 = 5 };

/* FP8 E4M3 code -> exact double.  The OCP "e4m3fn" layout: sign, 4 exponent
 * bits (bias 7), 3 mantissa bits; exponent field 0 holds the subnormals
 * m * 2^-9; S.1111.111 is NaN; there is no infinity and the largest finite
 * value is 1.75 * 2^8 = 448, the limit [LatentMoE] compares the SiTU-GLU
 * product bound with. */
double or_e4m3_to_f64(uint8_t c) {
  int sign = c >> 7, ex = (c >> 3) & 0xF, man = c & 7;
  double v;
  if (ex == 15 && man == 7) return NAN;
  if (ex == 0) {
    v = ldexp((double)man, -9);
  } else {
    v = ldexp((double)(8 + man), ex - 10);
  }
  return sign ? -v : v;
}

/* Nearest E4M3 code to x, ties to the even code (even mantissa), among the
 * 127 finite magnitudes (codes 0x00..0x7E, increasing with the code);
 * magnitudes above 448 give 448 (saturation, the "satfinite" conversion),
 * NaN gives the NaN code, the sign of x (also of a zero result) is kept.
 * The search is a bisection for the largest magnitude not above |x| in the
 * table of decoded magnitudes, then the nearer of it and the next one. */
static double e4m3_mag[127];

__attribute__((constructor)) static void e4m3_mag_fill(void) { /* at library load */
  for (int c = 0; c <= 0x7E; ++c) e4m3_mag[c] = or_e4m3_to_f64((uint8_t)c);
}

uint8_t or_round_e4m3(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  if (isinf(x)) return (uint8_t)(sign | 0x7E); /* saturates like any magnitude above 448 */
  double a = fabs(x);
  if (a >= e4m3_mag[0x7E]) return (uint8_t)(sign | 0x7E);
  int lo = 0, hi = 0x7E; /* e4m3_mag[lo] <= a < e4m3_mag[hi] */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (e4m3_mag[mid] <= a) lo = mid; else hi = mid;
  }
  double dlo = a - e4m3_mag[lo], dhi = e4m3_mag[hi] - a;
  int best = dlo < dhi ? lo : dhi < dlo ? hi : ((lo & 1) == 0 ? lo : hi);
  return (uint8_t)(sign | best);
}

/* Row-wise E4M3 quantisation of an fp32 [rows][cols] matrix: per row
 * s = amax / 448 (one fp32 division; s = 1 for an all-zero row) and
 * code = nearest E4M3 of the fp32 quotient x / s, so that s * e4m3(code)
 * approximates x and the row's largest magnitude maps to +-448. */
void or_quant_e4m3_rows(int64_t rows, int64_t cols, const float* x, uint8_t* codes,
                        float* scales) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    float amax = 0.0f;
    for (int64_t c = 0; c < cols; ++c) amax = fmaxf(amax, fabsf(x[r * cols + c]));
    const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    scales[r] = s;
    for (int64_t c = 0; c < cols; ++c) {
      const float q = x[r * cols + c] / s;
      codes[r * cols + c] = or_round_e4m3((double)q);
    }
  }
}

/* One [rows][cols] matrix in any storage type.  q4_0 (format named in
 * [MCU #13] §4): blocks of 32 consecutive values along a row, one fp16 scale
 * s per block, 4-bit codes q in 0..15, value (q - 8) * s; byte j (0..15) of a
 * block holds element j in its low nibble and element j + 16 in its high
 * nibble. */
typedef struct {
  int dtype;
  int64_t rows, cols;
  const void* data;       /* f32 / bf16 / f16 / f64 */
  const uint8_t* qs;      /* q4_0: [rows][cols/2] */
  const uint16_t* scales; /* q4_0: [rows][cols/32] fp16 codes */
  const float* row_scale; /* e4m3: [rows] fp32, value = row_scale[r] * e4m3(data[r][c]) */
} or_mat;

static inline double mat_get(const or_mat* m, int64_t r, int64_t c) {
  switch (m->dtype) {
    case OR_F32: return (double)((const float*)m->data)[r * m->cols + c];
    case OR_BF16: return or_bf16_to_f64(((const uint16_t*)m->data)[r * m->cols + c]);
    case OR_F16: return or_f16_to_f64(((const uint16_t*)m->data)[r * m->cols + c]);
    case OR_F64: return ((const double*)m->data)[r * m->cols + c];
    case OR_E4M3:
      return (double)m->row_scale[r] * or_e4m3_to_f64(((const uint8_t*)m->data)[r * m->cols + c]);
    default: {
      int64_t b = c / 32, j = c % 32;
      uint8_t byte = m->qs[r * (m->cols / 2) + b * 16 + (j & 15)];
      int q = (j < 16) ? (byte & 0xF) : (byte >> 4);
      return (double)(q - 8) * or_f16_to_f64(m->scales[r * (m->cols / 32) + b]);
    }
  }
}

/* Decode a whole matrix (or vector) to double. */
void or_mat_decode(const or_mat* m, double* out) {
  for (int64_t r = 0; r < m->rows; ++r)
    for (int64_t c = 0; c < m->cols; ++c) out[r * m->cols + c] = mat_get(m, r, c);
}

/* Round a double to the nearest bf16 value through fp32 (the storage a GPU
 * kernel uses for an intermediate it writes as bf16), returned as double. */
double or_round_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  u &= 0xFFFF0000u;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Element-wise or_round_bf16 over n values. */
void or_round_bf16_n(int64_t n, const double* x, double* y) {
  for (int64_t i = 0; i < n; ++i) y[i] = or_round_bf16(x[i]);
}

/* Round a double to the nearest IEEE binary16 (ties to even) and return its
 * bit pattern: the storage of the fp16 decode activations between layers. */
uint16_t or_round_f16(double x) {
  _Float16 h = (_Float16)x;
  uint16_t u;
  memcpy(&u, &h, 2);
  return u;
}

/* ------------------------------------------------------------------- router */

/* Router logit z = (W_route u)_i  [MoE tutorial] §3.2, formed in fp32.
 * The page fixes fp32 but not the summation order.  The order used is a
 * blocked sum: the input index is cut into blocks of OR_ROUTER_BLOCK = 128
 * consecutive elements (the last block may be shorter); each block's partial
 * sum P_m is a chain of fused multiply-adds (one rounding each) over its
 * elements in ascending order, starting from +0; z is then +0 plus P_0, plus
 * P_1, ... in ascending block order, each addition rounded in fp32.  For
 * d <= 128 this is the plain ascending chain. */
enum { OR_ROUTER_BLOCK = 128 };

float or_router_logit(const float* w, const float* u, int64_t d) {
  float z = 0.0f;
  for (int64_t j0 = 0; j0 < d; j0 += OR_ROUTER_BLOCK) {
    const int64_t j1 = j0 + OR_ROUTER_BLOCK < d ? j0 + OR_ROUTER_BLOCK : d;
    float part = 0.0f;
    for (int64_t j = j0; j < j1; ++j) part = fmaf(w[j], u[j], part);
    z = z + part;
  }
  return z;
}

/* Routing of T tokens  [MoE tutorial] §3.2:
 *   z_{t,i} = (W_route u_t)_i (+ b_i),  p = softmax(z),
 *   S_t = the k experts with the largest z (ties: lower expert index),
 *   a_{t,i} = p_{t,i} / sum_{j in S_t} p_{t,j}  (renorm = 1, Mixtral style) or
 *   a_{t,i} = p_{t,i} (renorm = 0, the top-1 Switch multiplier of §3.2).
 * Selection by z equals selection by p (softmax is monotone) without the ties
 * that rounding p could introduce.  Outputs: logits [T][N] fp32, probs and
 * top_w in double, top_idx [T][k] ordered by descending z. */
void or_route(int64_t T, int64_t d, int64_t N, int64_t k, int renorm, const float* u,
              const float* w_route, const float* bias, float* logits, double* probs,
              int32_t* top_idx, double* top_w) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t t = 0; t < T; ++t) {
    float* z = logits + t * N;
    for (int64_t i = 0; i < N; ++i) {
      z[i] = or_router_logit(w_route + i * d, u + t * d, d);
      if (bias) z[i] = z[i] + bias[i];
    }
    double zmax = -INFINITY;
    for (int64_t i = 0; i < N; ++i) zmax = fmax(zmax, (double)z[i]);
    double den = 0.0;
    for (int64_t i = 0; i < N; ++i) den += exp((double)z[i] - zmax);
    double* p = probs + t * N;
    for (int64_t i = 0; i < N; ++i) p[i] = exp((double)z[i] - zmax) / den;
    /* top-k by repeated selection of the best remaining (z desc, index asc) */
    int32_t* sel = top_idx + t * k;
    for (int64_t s = 0; s < k; ++s) {
      int64_t best = -1;
      for (int64_t i = 0; i < N; ++i) {
        int taken = 0;
        for (int64_t q = 0; q < s; ++q) taken |= (sel[q] == i);
        if (taken) continue;
        if (best < 0 || z[i] > z[best]) best = i;
      }
      sel[s] = (int32_t)best;
    }
    double ssum = 0.0;
    for (int64_t s = 0; s < k; ++s) ssum += p[sel[s]];
    for (int64_t s = 0; s < k; ++s) top_w[t * k + s] = renorm ? p[sel[s]] / ssum : p[sel[s]];
  }
}

/* The same routing from given logits (the tutorial's controlled-logit
 * experiments feed logits directly).  No fp32 dot product involved. */
void or_route_from_logits(int64_t T, int64_t N, int64_t k, int renorm, const float* logits,
                          double* probs, int32_t* top_idx, double* top_w) {
  for (int64_t t = 0; t < T; ++t) {
    const float* z = logits + t * N;
    double zmax = -INFINITY, den = 0.0;
    for (int64_t i = 0; i < N; ++i) zmax = fmax(zmax, (double)z[i]);
    for (int64_t i = 0; i < N; ++i) den += exp((double)z[i] - zmax);
    for (int64_t i = 0; i < N; ++i) probs[t * N + i] = exp((double)z[i] - zmax) / den;
    int32_t* sel = top_idx + t * k;
    for (int64_t s = 0; s < k; ++s) {
      int64_t best = -1;
      for (int64_t i = 0; i < N; ++i) {
        int taken = 0;
        for (int64_t q = 0; q < s; ++q) taken |= (sel[q] == i);
        if (!taken && (best < 0 || z[i] > z[best])) best = i;
      }
      sel[s] = (int32_t)best;
    }
    double ssum = 0.0;
    for (int64_t s = 0; s < k; ++s) ssum += probs[t * N + sel[s]];
    for (int64_t s = 0; s < k; ++s)
      top_w[t * k + s] = renorm ? probs[t * N + sel[s]] / ssum : probs[t * N + sel[s]];
  }
}

/* --------------------------------------------------------------- aux stats */

/* Switch balancing statistics  [MoE tutorial] §3.4:
 *   f_i = (1/T) #{t : argmax_j p_{t,j} = i}   (argmax = slot 0 of the top-k)
 *   P_i = (1/T) sum_t p_{t,i}
 *   n_sum_fP = N * sum_i f_i P_i               (L_aux without alpha)
 * plus the dispatch loads L_i = #{(t,s) : top_idx[t][s] = i}  (§3.6). */
void or_aux_stats(int64_t T, int64_t N, int64_t k, const double* probs, const int32_t* top_idx,
                  double* f, double* P, double* n_sum_fP, int32_t* loads) {
  for (int64_t i = 0; i < N; ++i) {
    f[i] = 0.0;
    P[i] = 0.0;
    loads[i] = 0;
  }
  for (int64_t t = 0; t < T; ++t) {
    f[top_idx[t * k]] += 1.0;
    for (int64_t s = 0; s < k; ++s) loads[top_idx[t * k + s]] += 1;
    for (int64_t i = 0; i < N; ++i) P[i] += probs[t * N + i];
  }
  double acc = 0.0;
  for (int64_t i = 0; i < N; ++i) {
    f[i] /= (double)T;
    P[i] /= (double)T;
    acc += f[i] * P[i];
  }
  *n_sum_fP = (double)N * acc;
}

/* -------------------------------------------------------- capacity, permute */

/* Expert capacity C = ceil(c * T / N)  [MoE tutorial] §3.5, with T counted as
 * dispatches (k * T) for top-k as §3.5 requires. */
int64_t or_capacity(int64_t T, int64_t N, int64_t k, double factor) {
  return (int64_t)ceil(factor * (double)(k * T) / (double)N);
}

/* Group dispatches by expert  [MoE tutorial] §3.5, §3.6, §3.8.
 * Dispatch (t, s) goes to expert top_idx[t][s].  Its rank is the number of
 * dispatches to the same expert from lower token indices.  It is kept when
 * C == 0 (unlimited) or rank < C; a dropped dispatch skips the expert
 * (the residual path carries the token).  Grouped row of a kept dispatch:
 * offsets[e] + rank, where offsets is the exclusive prefix sum of the kept
 * counts.  Outputs:
 *   counts[e]   = L_e (all dispatches, kept or not)
 *   offsets[N+1]
 *   perm_tok[r] = token of grouped row r   (r < offsets[N])
 *   row_of[t][s] = grouped row, or -1 if dropped
 *   overflow[e] = max(L_e - C, 0)
 *   totals = {kept, sum overflow, sum empty slots max(C - L_e, 0)} */
void or_permute(int64_t T, int64_t N, int64_t k, int64_t C, const int32_t* top_idx,
                int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                int32_t* overflow, int64_t* totals) {
  int64_t* seen = (int64_t*)calloc((size_t)N, sizeof(int64_t));
  for (int64_t e = 0; e < N; ++e) counts[e] = 0;
  for (int64_t x = 0; x < T * k; ++x) counts[top_idx[x]] += 1;
  int64_t run = 0, of = 0, empty = 0;
  for (int64_t e = 0; e < N; ++e) {
    offsets[e] = (int32_t)run;
    int64_t kept = (C > 0 && counts[e] > C) ? C : counts[e];
    run += kept;
    overflow[e] = (int32_t)((C > 0 && counts[e] > C) ? counts[e] - C : 0);
    of += overflow[e];
    empty += (C > 0 && counts[e] < C) ? C - counts[e] : 0;
  }
  offsets[N] = (int32_t)run;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t s = 0; s < k; ++s) {
      int32_t e = top_idx[t * k + s];
      int64_t rank = seen[e]++;
      if (C > 0 && rank >= C) {
        row_of[t * k + s] = -1;
      } else {
        int64_t r = offsets[e] + rank;
        row_of[t * k + s] = (int32_t)r;
        perm_tok[r] = (int32_t)t;
      }
    }
  }
  totals[0] = run;
  totals[1] = of;
  totals[2] = empty;
  free(seen);
}

/* ------------------------------------------------------------ expert FFN */

/* y = W x for one [rows][cols] matrix, in double. */
void or_matvec(const or_mat* W, const double* x, double* y) {
  for (int64_t r = 0; r < W->rows; ++r) {
    double acc = 0.0;
    for (int64_t c = 0; c < W->cols; ++c) acc += mat_get(W, r, c) * x[c];
    y[r] = acc;
  }
}

static inline double silu(double g) { return g / (1.0 + exp(-g)); }

/* One expert F(u) = W_down (SiLU(W_gate u) (*) W_up u)  [MoE tutorial] §3.1.
 * act = 1 applies the SiTU-GLU soft caps of [LatentMoE]: the gate and up
 * pre-activations become beta_g tanh(g / beta_g) and beta_u tanh(u / beta_u)
 * before SiLU and the product.  round_h = 1 rounds the hidden vector to bf16
 * (the storage of the intermediate in the bf16 layers), round_h = 2 to FP8
 * E4M3 with no scale (the FP8 experts: the soft caps keep |H| below
 * beta_g * beta_u = 100 < 448, so H needs no per-row scale).  W_gate, W_up:
 * [h][d_in]; W_down: [d_out][h]. */
void or_expert(const or_mat* Wg, const or_mat* Wu, const or_mat* Wd, const double* u, int act,
               double beta_g, double beta_u, int round_h, double* out) {
  int64_t h = Wg->rows;
  double* g = (double*)malloc(sizeof(double) * (size_t)h);
  double* v = (double*)malloc(sizeof(double) * (size_t)h);
  or_matvec(Wg, u, g);
  or_matvec(Wu, u, v);
  for (int64_t i = 0; i < h; ++i) {
    double gi = g[i], ui = v[i];
    if (act == 1) {
      gi = beta_g * tanh(gi / beta_g);
      ui = beta_u * tanh(ui / beta_u);
    }
    double hi = silu(gi) * ui;
    g[i] = round_h == 1 ? or_round_bf16(hi)
           : round_h == 2 ? or_e4m3_to_f64(or_round_e4m3(hi))
                          : hi;
  }
  or_matvec(Wd, g, out);
  free(g);
  free(v);
}

/* Token outputs of the sparse layer  [MoE tutorial] §3.2:
 *   y_t = sum over kept dispatches s of a_{t,s} F_{top_idx[t][s]}(u_t);
 * a dropped dispatch (row_of = -1) contributes nothing and the remaining
 * weights are not renormalised.  Experts are [N] arrays of matrices.  Only
 * the n_sel tokens listed in tokens[] are evaluated (all of them when the
 * caller lists every token).  u is [T][d_in] in double. */
void or_moe_tokens(int64_t k, const or_mat* Wg, const or_mat* Wu, const or_mat* Wd,
                   const double* u, int64_t d_in, const int32_t* top_idx, const double* top_w,
                   const int32_t* row_of, int act, double beta_g, double beta_u, int round_h,
                   const int32_t* tokens, int64_t n_sel, double* y) {
  int64_t d_out = Wd[0].rows;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t q = 0; q < n_sel; ++q) {
    int64_t t = tokens[q];
    double* acc = y + q * d_out;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)d_out);
    for (int64_t m = 0; m < d_out; ++m) acc[m] = 0.0;
    for (int64_t s = 0; s < k; ++s) {
      if (row_of && row_of[t * k + s] < 0) continue;
      int32_t e = top_idx[t * k + s];
      or_expert(&Wg[e], &Wu[e], &Wd[e], u + t * d_in, act, beta_g, beta_u, round_h, tmp);
      for (int64_t m = 0; m < d_out; ++m) acc[m] += top_w[t * k + s] * tmp[m];
    }
    free(tmp);
  }
}

/* Weighted combine of per-row expert outputs  [MoE tutorial] §3.2 eq. y and
 * §3.6 (results added back to [T, d] by token index): for each token,
 * y_t = sum over slots s with row_of[t][s] >= 0 of top_w[t][s] * rows[row_of[t][s]]. */
void or_combine(int64_t T, int64_t k, int64_t width, const double* rows, const int32_t* row_of,
                const double* top_w, double* y) {
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t m = 0; m < width; ++m) y[t * width + m] = 0.0;
    for (int64_t s = 0; s < k; ++s) {
      int32_t r = row_of[t * k + s];
      if (r < 0) continue;
      for (int64_t m = 0; m < width; ++m) y[t * width + m] += top_w[t * k + s] * rows[r * width + m];
    }
  }
}

/* Dense brute-force reference  [MoE tutorial] appendix lab: every expert is
 * evaluated for every token and multiplied by its combine weight, which is
 * zero for the unselected experts.  Must equal or_moe_tokens exactly when
 * nothing is dropped. */
void or_moe_dense(int64_t T, int64_t N, int64_t k, const or_mat* Wg, const or_mat* Wu,
                  const or_mat* Wd, const double* u, int64_t d_in, const int32_t* top_idx,
                  const double* top_w, int act, double beta_g, double beta_u, int round_h,
                  double* y) {
  int64_t d_out = Wd[0].rows;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    double* tmp = (double*)malloc(sizeof(double) * (size_t)d_out);
    for (int64_t m = 0; m < d_out; ++m) y[t * d_out + m] = 0.0;
    for (int64_t e = 0; e < N; ++e) {
      double w = 0.0;
      for (int64_t s = 0; s < k; ++s)
        if (top_idx[t * k + s] == e) w += top_w[t * k + s];
      or_expert(&Wg[e], &Wu[e], &Wd[e], u + t * d_in, act, beta_g, beta_u, round_h, tmp);
      for (int64_t m = 0; m < d_out; ++m) y[t * d_out + m] += w * tmp[m];
    }
    free(tmp);
  }
}

/* RMSNorm without gain  [LatentMoE]: x / sqrt(mean(x^2) + eps). */
void or_rmsnorm(int64_t n, const double* x, double eps, double* y) {
  double ss = 0.0;
  for (int64_t i = 0; i < n; ++i) ss += x[i] * x[i];
  double r = sqrt(ss / (double)n + eps);
  for (int64_t i = 0; i < n; ++i) y[i] = x[i] / r;
}

/* ------------------------------------------------------------------ ledgers */

/* Expert parameter ledger  [MoE tutorial] §3.3 and §01:
 * one SwiGLU expert has 3dh weights; N experts 3dhN; k active 3dhk. */
void or_ledger(int64_t d, int64_t h, int64_t N, int64_t k, int64_t* one, int64_t* all,
               int64_t* active, double* bf16_gib) {
  *one = 3 * d * h;
  *all = N * *one;
  *active = k * *one;
  *bf16_gib = (double)(*all) * 2.0 / 1073741824.0;
}

/* Expert-weight bandwidth gain of top-k lookup-loading  [MCU #10] §3 table,
 * [MCU #13] §2: dense FFN width over the k selected expert widths. */
double or_bandwidth_gain(int64_t ffn, int64_t top_k, int64_t ffn_e) {
  return (double)ffn / (double)(top_k * ffn_e);
}

/* ------------------------------------------------------- quantile balancing */
/* [LatentMoE] Quantile Balancing.  With every token's top-k cutoff a_i held
 * fixed, expert j takes token i iff s_ij + b_j >= a_i, i.e. iff
 * b_j >= required_ij = a_i - s_ij; the bias that gives expert j exactly q
 * tokens is the q-th smallest required_ij, found in one step instead of a
 * fixed-step update.  The arithmetic is the router's fp32: the selection
 * score s_ij + b_j and required_ij = a_i - s_ij each round once. */

static int or_cmp_float_desc(const void* x, const void* y) {
  const float a = *(const float*)x, b = *(const float*)y;
  return (a < b) - (a > b);
}
static int or_cmp_float_asc(const void* x, const void* y) {
  const float a = *(const float*)x, b = *(const float*)y;
  return (a > b) - (a < b);
}

/* a_i = the k-th largest selection score s_ij + b_j (b nullable = 0). */
void or_qb_cutoffs(int64_t T, int64_t N, int64_t k, const float* s, const float* b, float* a) {
  float* row = (float*)malloc((size_t)N * sizeof(float));
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < N; ++j) {
      const float v = s[t * N + j];
      row[j] = b ? v + b[j] : v;
    }
    qsort(row, (size_t)N, sizeof(float), or_cmp_float_desc);
    a[t] = row[k - 1];
  }
  free(row);
}

/* b_j = the q-th smallest (1-based) required_ij over the T tokens, a zero
 * returned as +0; loads_j = #{i : required_ij <= b_j} (q when the values are
 * distinct). */
void or_qb_exact(int64_t T, int64_t N, const float* s, const float* a, int64_t q, float* b_out,
                 int32_t* loads) {
  float* req = (float*)malloc((size_t)T * sizeof(float));
  float* srt = (float*)malloc((size_t)T * sizeof(float));
  for (int64_t j = 0; j < N; ++j) {
    for (int64_t i = 0; i < T; ++i) req[i] = a[i] - s[i * N + j];
    memcpy(srt, req, (size_t)T * sizeof(float));
    qsort(srt, (size_t)T, sizeof(float), or_cmp_float_asc);
    float v = srt[q - 1];
    if (v == 0.0f) v = 0.0f;
    b_out[j] = v;
    if (loads) {
      int32_t c = 0;
      for (int64_t i = 0; i < T; ++i) c += req[i] <= v;
      loads[j] = c;
    }
  }
  free(req);
  free(srt);
}

/* Histogram estimate of the same quantile: B equal bins over [lo, hi], the
 * smallest and largest required_ij of expert j; the bin of v is
 * min(B - 1, trunc((v - lo) * scale)) with scale = B / (hi - lo); the
 * estimate is the upper edge lo + (c + 1) * w of the first bin c at which the
 * running count reaches q, w = (hi - lo) / B.  Every step is one fp32
 * operation; hi == lo gives lo. */
void or_qb_hist(int64_t T, int64_t N, const float* s, const float* a, int64_t q, int64_t B,
                float* b_out) {
  float* req = (float*)malloc((size_t)T * sizeof(float));
  int64_t* cnt = (int64_t*)malloc((size_t)B * sizeof(int64_t));
  for (int64_t j = 0; j < N; ++j) {
    float lo = 0.0f, hi = 0.0f;
    for (int64_t i = 0; i < T; ++i) {
      req[i] = a[i] - s[i * N + j];
      if (i == 0 || req[i] < lo) lo = req[i];
      if (i == 0 || req[i] > hi) hi = req[i];
    }
    if (!(hi > lo)) {
      b_out[j] = lo == 0.0f ? 0.0f : lo;
      continue;
    }
    const float range = hi - lo;
    const float scale = (float)B / range;
    const float w = range / (float)B;
    for (int64_t c = 0; c < B; ++c) cnt[c] = 0;
    for (int64_t i = 0; i < T; ++i) {
      const float x = (req[i] - lo) * scale;
      int64_t c = (int64_t)x;
      if (c > B - 1) c = B - 1;
      ++cnt[c];
    }
    int64_t c = 0, cum = 0;
    for (; c < B; ++c) {
      cum += cnt[c];
      if (cum >= q) break;
    }
    if (c > B - 1) c = B - 1;
    const float edge = (float)(c + 1) * w;
    b_out[j] = lo + edge;
  }
  free(req);
  free(cnt);
}

/* ------------------------------------------------------ aux-loss gradient */
/* [MoE tutorial] §3.7: with the batch loads f held constant,
 * dL_aux/dz_tj = (alpha N / T) p_tj (f_j - sum_i f_i p_ti), in double. */
void or_aux_grad(int64_t T, int64_t N, double alpha, const double* p, const double* f,
                 double* dz) {
  const double c = alpha * (double)N / (double)T;
  for (int64_t t = 0; t < T; ++t) {
    double fbar = 0.0;
    for (int64_t i = 0; i < N; ++i) fbar += f[i] * p[t * N + i];
    for (int64_t j = 0; j < N; ++j) dz[t * N + j] = c * p[t * N + j] * (f[j] - fbar);
  }
}

/* ------------------------------------------------------- layer backward */
/* The loss whose gradient the backward pass forms:
 *   L = sum_t dy_t . y_t  +  alpha N sum_i f_i P_i      (second term when f != NULL)
 * y_t = sum over kept slots s of a_{t,s} F_{e_{t,s}}(u_t)   [MoE tutorial] §3.1, §3.2
 * p_t = softmax(z_t), z_t = W_route u_t (or the given z_t when W_route is NULL)
 * a_{t,s} = p_{t,e_{t,s}} / sum_r p_{t,e_{t,r}}  (renorm = 1; over all k slots,
 *           kept or dropped, as in the forward), or p_{t,e_{t,s}} (renorm = 0)
 * P_i = (1/T) sum_t p_{t,i}                               [MoE tutorial] §3.4
 * dy is the upstream gradient dL/dy.  The selected sets (top_idx) and the
 * dropped dispatches (row_of < 0) are inputs and are held fixed: top-k and the
 * capacity cut are piecewise constant in the parameters, so they contribute
 * no derivative; the loads f are held fixed as [MoE tutorial] §3.7 states.
 * Every quantity, the logits included, is in double: this is the exact-
 * arithmetic gradient, not a replay of the fp32 routing decision.  Only the
 * selected experts of kept dispatches receive weight gradient, the property
 * the [LatentMoE] demo tests ("only selected experts receive gradient"). */

/* Softmax of one row in double, max subtracted (as or_route_from_logits). */
static void or_softmax_row(int64_t N, const double* z, double* p) {
  double zmax = -INFINITY, den = 0.0;
  for (int64_t i = 0; i < N; ++i) zmax = fmax(zmax, z[i]);
  for (int64_t i = 0; i < N; ++i) den += exp(z[i] - zmax);
  for (int64_t i = 0; i < N; ++i) p[i] = exp(z[i] - zmax) / den;
}

/* z_t (W_route given: W_route u_t in double; else the given row), p_t, and
 * the combine weights a_t of the k slots. */
static void or_token_weights(int64_t N, int64_t d_in, int64_t k, int renorm, const double* Wr,
                             const double* z_in, const double* u, const int32_t* sel, double* z,
                             double* p, double* a) {
  for (int64_t j = 0; j < N; ++j) {
    if (Wr) {
      double acc = 0.0;
      for (int64_t c = 0; c < d_in; ++c) acc += Wr[j * d_in + c] * u[c];
      z[j] = acc;
    } else {
      z[j] = z_in[j];
    }
  }
  or_softmax_row(N, z, p);
  double ssum = 0.0;
  for (int64_t s = 0; s < k; ++s) ssum += p[sel[s]];
  for (int64_t s = 0; s < k; ++s) a[s] = renorm ? p[sel[s]] / ssum : p[sel[s]];
}

/* L above; y (nullable) receives y_t [T][d_out].  Wr [N][d_in] or NULL (then
 * z [T][N] is used); f [N] or NULL (no balancing term). */
double or_layer_loss(int64_t T, int64_t N, int64_t k, int renorm, const or_mat* Wg,
                     const or_mat* Wu, const or_mat* Wd, int act, double beta_g, double beta_u,
                     const double* Wr, const double* z, const double* u, int64_t d_in,
                     const int32_t* top_idx, const int32_t* row_of, const double* dy,
                     double alpha, const double* f, double* y) {
  int64_t d_out = Wd[0].rows;
  double* zt = (double*)malloc(sizeof(double) * (size_t)N);
  double* pt = (double*)malloc(sizeof(double) * (size_t)N);
  double* at = (double*)malloc(sizeof(double) * (size_t)k);
  double* F = (double*)malloc(sizeof(double) * (size_t)d_out);
  double* yt = (double*)malloc(sizeof(double) * (size_t)d_out);
  double* P = (double*)calloc((size_t)N, sizeof(double));
  double L = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    or_token_weights(N, d_in, k, renorm, Wr, z ? z + t * N : NULL, u + t * d_in, top_idx + t * k,
                     zt, pt, at);
    for (int64_t i = 0; i < N; ++i) P[i] += pt[i];
    for (int64_t m = 0; m < d_out; ++m) yt[m] = 0.0;
    for (int64_t s = 0; s < k; ++s) {
      if (row_of && row_of[t * k + s] < 0) continue;
      int32_t e = top_idx[t * k + s];
      or_expert(&Wg[e], &Wu[e], &Wd[e], u + t * d_in, act, beta_g, beta_u, 0, F);
      for (int64_t m = 0; m < d_out; ++m) yt[m] += at[s] * F[m];
    }
    for (int64_t m = 0; m < d_out; ++m) L += dy[t * d_out + m] * yt[m];
    if (y)
      for (int64_t m = 0; m < d_out; ++m) y[t * d_out + m] = yt[m];
  }
  if (f) {
    double acc = 0.0;
    for (int64_t i = 0; i < N; ++i) acc += f[i] * (P[i] / (double)T);
    L += alpha * (double)N * acc;
  }
  free(zt);
  free(pt);
  free(at);
  free(F);
  free(yt);
  free(P);
  return L;
}

static inline double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Backward of one expert evaluation F(u) = W_down (SiLU(g') (*) v'),
 * g = W_gate u, v = W_up u, g' = g and v' = v (act = 0) or the soft caps
 * beta tanh(x / beta) of [LatentMoE] (act = 1).  Given dF = dL/dF [d_out]:
 *   dH = W_down^T dF,            dW_down += dF H^T
 *   dg' = dH (*) v' (*) SiLU'(g'), SiLU'(x) = s(x) (1 + x (1 - s(x))), s = sigmoid
 *   dv' = dH (*) SiLU(g')
 *   dg = dg' (1 - tanh^2(g / beta_g)) under the cap, else dg'; the same for v
 *   dW_gate += dg u^T, dW_up += dv u^T, du += W_gate^T dg + W_up^T dv.
 * F(u) is returned in out.  Accumulators: dWg, dWu [h][d_in], dWd [d_out][h],
 * du [d_in]. */
static void or_expert_backward(const or_mat* Wg, const or_mat* Wu, const or_mat* Wd,
                               const double* u, int act, double beta_g, double beta_u,
                               const double* dF, double* out, double* dWg, double* dWu,
                               double* dWd, double* du) {
  int64_t h = Wg->rows, d_in = Wg->cols, d_out = Wd->rows;
  double* g = (double*)malloc(sizeof(double) * (size_t)h);
  double* v = (double*)malloc(sizeof(double) * (size_t)h);
  double* H = (double*)malloc(sizeof(double) * (size_t)h);
  double* dH = (double*)malloc(sizeof(double) * (size_t)h);
  or_matvec(Wg, u, g);
  or_matvec(Wu, u, v);
  for (int64_t i = 0; i < h; ++i) {
    double gc = act == 1 ? beta_g * tanh(g[i] / beta_g) : g[i];
    double vc = act == 1 ? beta_u * tanh(v[i] / beta_u) : v[i];
    H[i] = silu(gc) * vc;
  }
  or_matvec(Wd, H, out);
  for (int64_t i = 0; i < h; ++i) {
    double acc = 0.0;
    for (int64_t m = 0; m < d_out; ++m) acc += mat_get(Wd, m, i) * dF[m];
    dH[i] = acc;
  }
  for (int64_t m = 0; m < d_out; ++m)
    for (int64_t i = 0; i < h; ++i) dWd[m * h + i] += dF[m] * H[i];
  for (int64_t i = 0; i < h; ++i) {
    double gc = g[i], vc = v[i], jg = 1.0, jv = 1.0;
    if (act == 1) {
      double tg = tanh(g[i] / beta_g), tv = tanh(v[i] / beta_u);
      gc = beta_g * tg;
      vc = beta_u * tv;
      jg = 1.0 - tg * tg;
      jv = 1.0 - tv * tv;
    }
    double sg = sigmoid(gc);
    double dg = dH[i] * vc * (sg * (1.0 + gc * (1.0 - sg))) * jg;
    double dv = dH[i] * silu(gc) * jv;
    for (int64_t c = 0; c < d_in; ++c) {
      dWg[i * d_in + c] += dg * u[c];
      dWu[i * d_in + c] += dv * u[c];
      du[c] += mat_get(Wg, i, c) * dg + mat_get(Wu, i, c) * dv;
    }
  }
  free(g);
  free(v);
  free(H);
  free(dH);
}

/* dL/d(everything) for L of or_layer_loss, with the same inputs.
 * Per token t (a_s, p from or_token_weights):
 *   kept slot s, expert e:  da_s = dy_t . F_e(u_t); the expert backward with
 *                           dF = a_s dy_t adds to dW*_e and du_t
 *   dropped slot:           da_s = 0 (it contributes nothing to y_t)
 *   renorm:                 dp_{e_s} = (da_s - sum_r a_r da_r) / sum_r p_{e_r}
 *   no renorm:              dp_{e_s} = da_s;  dp_i = 0 outside the selected set
 *   softmax:                dz_j = p_j (dp_j - sum_i p_i dp_i)
 *   balancing term:         dz_j += (alpha N / T) p_j (f_j - sum_i f_i p_i)  (§3.7)
 *   router (Wr given):      dWr_j += dz_j u_t,  du_t += sum_j dz_j Wr_j
 * Outputs (fully overwritten): dz [T][N], du [T][d_in], dWr [N][d_in] (only
 * when Wr is given; may be NULL), dWg, dWu [N][h][d_in], dWd [N][d_out][h]. */
void or_layer_backward(int64_t T, int64_t N, int64_t k, int renorm, const or_mat* Wg,
                       const or_mat* Wu, const or_mat* Wd, int act, double beta_g,
                       double beta_u, const double* Wr, const double* z, const double* u,
                       int64_t d_in, const int32_t* top_idx, const int32_t* row_of,
                       const double* dy, double alpha, const double* f, double* dz, double* du,
                       double* dWr, double* dWg, double* dWu, double* dWd) {
  int64_t h = Wg[0].rows, d_out = Wd[0].rows;
  memset(du, 0, sizeof(double) * (size_t)(T * d_in));
  memset(dWg, 0, sizeof(double) * (size_t)(N * h * d_in));
  memset(dWu, 0, sizeof(double) * (size_t)(N * h * d_in));
  memset(dWd, 0, sizeof(double) * (size_t)(N * d_out * h));
  if (Wr && dWr) memset(dWr, 0, sizeof(double) * (size_t)(N * d_in));
  double* zt = (double*)malloc(sizeof(double) * (size_t)N);
  double* pt = (double*)malloc(sizeof(double) * (size_t)N);
  double* dp = (double*)malloc(sizeof(double) * (size_t)N);
  double* at = (double*)malloc(sizeof(double) * (size_t)k);
  double* da = (double*)malloc(sizeof(double) * (size_t)k);
  double* dF = (double*)malloc(sizeof(double) * (size_t)d_out);
  double* F = (double*)malloc(sizeof(double) * (size_t)d_out);
  for (int64_t t = 0; t < T; ++t) {
    const double* ut = u + t * d_in;
    const double* dyt = dy + t * d_out;
    const int32_t* sel = top_idx + t * k;
    double* dut = du + t * d_in;
    double* dzt = dz + t * N;
    or_token_weights(N, d_in, k, renorm, Wr, z ? z + t * N : NULL, ut, sel, zt, pt, at);
    for (int64_t s = 0; s < k; ++s) {
      da[s] = 0.0;
      if (row_of && row_of[t * k + s] < 0) continue;
      int32_t e = sel[s];
      for (int64_t m = 0; m < d_out; ++m) dF[m] = at[s] * dyt[m];
      or_expert_backward(&Wg[e], &Wu[e], &Wd[e], ut, act, beta_g, beta_u, dF, F,
                         dWg + (int64_t)e * h * d_in, dWu + (int64_t)e * h * d_in,
                         dWd + (int64_t)e * d_out * h, dut);
      double acc = 0.0;
      for (int64_t m = 0; m < d_out; ++m) acc += dyt[m] * F[m];
      da[s] = acc;
    }
    for (int64_t i = 0; i < N; ++i) dp[i] = 0.0;
    if (renorm) {
      double ssum = 0.0, ada = 0.0;
      for (int64_t s = 0; s < k; ++s) {
        ssum += pt[sel[s]];
        ada += at[s] * da[s];
      }
      for (int64_t s = 0; s < k; ++s) dp[sel[s]] = (da[s] - ada) / ssum;
    } else {
      for (int64_t s = 0; s < k; ++s) dp[sel[s]] = da[s];
    }
    double pdp = 0.0;
    for (int64_t i = 0; i < N; ++i) pdp += pt[i] * dp[i];
    for (int64_t j = 0; j < N; ++j) dzt[j] = pt[j] * (dp[j] - pdp);
    if (f) {
      const double c = alpha * (double)N / (double)T;
      double fbar = 0.0;
      for (int64_t i = 0; i < N; ++i) fbar += f[i] * pt[i];
      for (int64_t j = 0; j < N; ++j) dzt[j] += c * pt[j] * (f[j] - fbar);
    }
    if (Wr) {
      for (int64_t j = 0; j < N; ++j) {
        for (int64_t c = 0; c < d_in; ++c) {
          if (dWr) dWr[j * d_in + c] += dzt[j] * ut[c];
          dut[c] += dzt[j] * Wr[j * d_in + c];
        }
      }
    }
  }
  free(zt);
  free(pt);
  free(dp);
  free(at);
  free(da);
  free(dF);
  free(F);
}

/* ------------------------------------------------ LatentMoE layer backward */
/* The LatentMoE layer of [LatentMoE] (width separation, RMSNorm before the
 * up-projection, SiTU-GLU routed experts, plain SwiGLU shared experts), in
 * double with no intermediate rounding, for one token x (width d):
 *   z = W_route x,  p = softmax(z),  a over the selected set (renorm or not)
 *   x_l = W_dp x                                  (width l)
 *   m = sum_s a_s E_{e_s}(x_l)                    (SiTU-GLU experts, width l)
 *   r = sqrt(mean(m^2) + eps),  m^ = m / r
 *   y = W_upp m^ + sum_j S_j(x)                   (width d)
 * and L = sum_t dy_t . y_t.  The selected sets are inputs held fixed. */
static void or_latent_token(int64_t N, int64_t k, int renorm, const or_mat* Wg,
                            const or_mat* Wu, const or_mat* Wd, double beta_g, double beta_u,
                            const double* Wr, const or_mat* Wdp, const or_mat* Wupp,
                            int64_t n_shared, const or_mat* Sg, const or_mat* Su,
                            const or_mat* Sd, double eps, const double* x, int64_t d,
                            const int32_t* sel, double* z, double* p, double* a, double* xl,
                            double* m, double* mh, double* r_out, double* y) {
  int64_t l = Wdp->rows;
  double* F = (double*)malloc(sizeof(double) * (size_t)(l > d ? l : d));
  or_token_weights(N, d, k, renorm, Wr, NULL, x, sel, z, p, a);
  or_matvec(Wdp, x, xl);
  for (int64_t i = 0; i < l; ++i) m[i] = 0.0;
  for (int64_t s = 0; s < k; ++s) {
    int32_t e = sel[s];
    or_expert(&Wg[e], &Wu[e], &Wd[e], xl, 1, beta_g, beta_u, 0, F);
    for (int64_t i = 0; i < l; ++i) m[i] += a[s] * F[i];
  }
  double ss = 0.0;
  for (int64_t i = 0; i < l; ++i) ss += m[i] * m[i];
  double r = sqrt(ss / (double)l + eps);
  for (int64_t i = 0; i < l; ++i) mh[i] = m[i] / r;
  *r_out = r;
  or_matvec(Wupp, mh, y);
  for (int64_t j = 0; j < n_shared; ++j) {
    or_expert(&Sg[j], &Su[j], &Sd[j], x, 0, 0.0, 0.0, 0, F);
    for (int64_t c = 0; c < d; ++c) y[c] += F[c];
  }
  free(F);
}

/* L = sum_t dy_t . y_t of the LatentMoE layer above; y (nullable) [T][d].
 * Routed experts: W_gate, W_up [h][l], W_down [l][h]; W_dp [l][d];
 * W_upp [d][l]; shared experts [sh][d], [d][sh]; W_route [N][d] double. */
double or_latent_loss(int64_t T, int64_t N, int64_t k, int renorm, const or_mat* Wg,
                      const or_mat* Wu, const or_mat* Wd, double beta_g, double beta_u,
                      const double* Wr, const or_mat* Wdp, const or_mat* Wupp, int64_t n_shared,
                      const or_mat* Sg, const or_mat* Su, const or_mat* Sd, double eps,
                      const double* x, int64_t d, const int32_t* top_idx, const double* dy,
                      double* y) {
  int64_t l = Wdp->rows;
  double* z = (double*)malloc(sizeof(double) * (size_t)N);
  double* p = (double*)malloc(sizeof(double) * (size_t)N);
  double* a = (double*)malloc(sizeof(double) * (size_t)k);
  double* xl = (double*)malloc(sizeof(double) * (size_t)l);
  double* m = (double*)malloc(sizeof(double) * (size_t)l);
  double* mh = (double*)malloc(sizeof(double) * (size_t)l);
  double* yt = (double*)malloc(sizeof(double) * (size_t)d);
  double L = 0.0, r;
  for (int64_t t = 0; t < T; ++t) {
    or_latent_token(N, k, renorm, Wg, Wu, Wd, beta_g, beta_u, Wr, Wdp, Wupp, n_shared, Sg, Su,
                    Sd, eps, x + t * d, d, top_idx + t * k, z, p, a, xl, m, mh, &r, yt);
    for (int64_t c = 0; c < d; ++c) L += dy[t * d + c] * yt[c];
    if (y)
      for (int64_t c = 0; c < d; ++c) y[t * d + c] = yt[c];
  }
  free(z);
  free(p);
  free(a);
  free(xl);
  free(m);
  free(mh);
  free(yt);
  return L;
}

/* Gradients of or_latent_loss.  Per token:
 *   dW_upp += dy m^T,  dm^ = W_upp^T dy
 *   RMSNorm:  dm = dm^ / r - m (sum_i dm^_i m_i) / (l r^3)
 *   routed slot s (expert e):  da_s = dm . E_e(x_l); the expert backward
 *       (soft caps included) with dF = a_s dm adds to dW*_e and dx_l
 *   renorm / softmax / router as in or_layer_backward: dz, dW_route += dz x^T,
 *       dx += W_route^T dz
 *   dW_dp += dx_l x^T,  dx += W_dp^T dx_l
 *   shared expert j: the SwiGLU backward with dF = dy adds to dS*_j and dx.
 * Outputs, all overwritten: dz [T][N], dx [T][d], dWr [N][d], dWdp [l][d],
 * dWupp [d][l], dWg, dWu [N][h][l], dWd [N][l][h], dSg, dSu [n][sh][d],
 * dSd [n][d][sh] (the shared ones may be NULL when n_shared = 0). */
void or_latent_backward(int64_t T, int64_t N, int64_t k, int renorm, const or_mat* Wg,
                        const or_mat* Wu, const or_mat* Wd, double beta_g, double beta_u,
                        const double* Wr, const or_mat* Wdp, const or_mat* Wupp,
                        int64_t n_shared, const or_mat* Sg, const or_mat* Su, const or_mat* Sd,
                        double eps, const double* x, int64_t d, const int32_t* top_idx,
                        const double* dy, double* dz, double* dx, double* dWr, double* dWdp,
                        double* dWupp, double* dWg, double* dWu, double* dWd, double* dSg,
                        double* dSu, double* dSd) {
  int64_t l = Wdp->rows, h = Wg[0].rows, sh = n_shared > 0 ? Sg[0].rows : 0;
  memset(dx, 0, sizeof(double) * (size_t)(T * d));
  memset(dWr, 0, sizeof(double) * (size_t)(N * d));
  memset(dWdp, 0, sizeof(double) * (size_t)(l * d));
  memset(dWupp, 0, sizeof(double) * (size_t)(d * l));
  memset(dWg, 0, sizeof(double) * (size_t)(N * h * l));
  memset(dWu, 0, sizeof(double) * (size_t)(N * h * l));
  memset(dWd, 0, sizeof(double) * (size_t)(N * l * h));
  if (n_shared > 0) {
    memset(dSg, 0, sizeof(double) * (size_t)(n_shared * sh * d));
    memset(dSu, 0, sizeof(double) * (size_t)(n_shared * sh * d));
    memset(dSd, 0, sizeof(double) * (size_t)(n_shared * d * sh));
  }
  double* z = (double*)malloc(sizeof(double) * (size_t)N);
  double* p = (double*)malloc(sizeof(double) * (size_t)N);
  double* dp = (double*)malloc(sizeof(double) * (size_t)N);
  double* a = (double*)malloc(sizeof(double) * (size_t)k);
  double* da = (double*)malloc(sizeof(double) * (size_t)k);
  double* xl = (double*)malloc(sizeof(double) * (size_t)l);
  double* dxl = (double*)malloc(sizeof(double) * (size_t)l);
  double* m = (double*)malloc(sizeof(double) * (size_t)l);
  double* mh = (double*)malloc(sizeof(double) * (size_t)l);
  double* dmh = (double*)malloc(sizeof(double) * (size_t)l);
  double* dm = (double*)malloc(sizeof(double) * (size_t)l);
  double* dF = (double*)malloc(sizeof(double) * (size_t)(l > d ? l : d));
  double* F = (double*)malloc(sizeof(double) * (size_t)(l > d ? l : d));
  double* yt = (double*)malloc(sizeof(double) * (size_t)d);
  for (int64_t t = 0; t < T; ++t) {
    const double* xt = x + t * d;
    const double* dyt = dy + t * d;
    const int32_t* sel = top_idx + t * k;
    double* dxt = dx + t * d;
    double* dzt = dz + t * N;
    double r;
    or_latent_token(N, k, renorm, Wg, Wu, Wd, beta_g, beta_u, Wr, Wdp, Wupp, n_shared, Sg, Su,
                    Sd, eps, xt, d, sel, z, p, a, xl, m, mh, &r, yt);
    /* up-projection and RMSNorm */
    for (int64_t i = 0; i < l; ++i) {
      double acc = 0.0;
      for (int64_t c = 0; c < d; ++c) acc += mat_get(Wupp, c, i) * dyt[c];
      dmh[i] = acc;
    }
    for (int64_t c = 0; c < d; ++c)
      for (int64_t i = 0; i < l; ++i) dWupp[c * l + i] += dyt[c] * mh[i];
    double dot = 0.0;
    for (int64_t i = 0; i < l; ++i) dot += dmh[i] * m[i];
    for (int64_t i = 0; i < l; ++i) dm[i] = dmh[i] / r - m[i] * dot / ((double)l * r * r * r);
    /* routed experts */
    for (int64_t i = 0; i < l; ++i) dxl[i] = 0.0;
    for (int64_t s = 0; s < k; ++s) {
      int32_t e = sel[s];
      for (int64_t i = 0; i < l; ++i) dF[i] = a[s] * dm[i];
      or_expert_backward(&Wg[e], &Wu[e], &Wd[e], xl, 1, beta_g, beta_u, dF, F,
                         dWg + (int64_t)e * h * l, dWu + (int64_t)e * h * l,
                         dWd + (int64_t)e * l * h, dxl);
      double acc = 0.0;
      for (int64_t i = 0; i < l; ++i) acc += dm[i] * F[i];
      da[s] = acc;
    }
    /* combine weights, softmax, router */
    for (int64_t j = 0; j < N; ++j) dp[j] = 0.0;
    if (renorm) {
      double ssum = 0.0, ada = 0.0;
      for (int64_t s = 0; s < k; ++s) {
        ssum += p[sel[s]];
        ada += a[s] * da[s];
      }
      for (int64_t s = 0; s < k; ++s) dp[sel[s]] = (da[s] - ada) / ssum;
    } else {
      for (int64_t s = 0; s < k; ++s) dp[sel[s]] = da[s];
    }
    double pdp = 0.0;
    for (int64_t j = 0; j < N; ++j) pdp += p[j] * dp[j];
    for (int64_t j = 0; j < N; ++j) dzt[j] = p[j] * (dp[j] - pdp);
    for (int64_t j = 0; j < N; ++j) {
      for (int64_t c = 0; c < d; ++c) {
        dWr[j * d + c] += dzt[j] * xt[c];
        dxt[c] += dzt[j] * Wr[j * d + c];
      }
    }
    /* down-projection into the latent width */
    for (int64_t i = 0; i < l; ++i) {
      for (int64_t c = 0; c < d; ++c) {
        dWdp[i * d + c] += dxl[i] * xt[c];
        dxt[c] += mat_get(Wdp, i, c) * dxl[i];
      }
    }
    /* shared experts at full width */
    for (int64_t j = 0; j < n_shared; ++j)
      or_expert_backward(&Sg[j], &Su[j], &Sd[j], xt, 0, 0.0, 0.0, dyt, F,
                         dSg + j * sh * d, dSu + j * sh * d, dSd + j * d * sh, dxt);
  }
  free(z);
  free(p);
  free(dp);
  free(a);
  free(da);
  free(xl);
  free(dxl);
  free(m);
  free(mh);
  free(dmh);
  free(dm);
  free(dF);
  free(F);
  free(yt);
}
