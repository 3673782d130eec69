// Shared helpers of the sm_100a MoE library: status reporting, number
// conversions, vector loads and host-side argument checks.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/moe.h"

namespace moe {

// ------------------------------------------------------- per-device caches
// Host-side values set up lazily once per device index (kernel attributes, SM
// counts, symbol addresses) live in static arrays of atomics, so host threads
// that make their first calls at the same time do not race.  Every such setup
// is idempotent, so two threads doing it once each is harmless.
constexpr int kMaxDevices = 64;

inline bool device_slot(int dev) { return dev >= 0 && dev < kMaxDevices; }

// SM count of the current device (cached per device; 148 if unknown).
int sm_count();

// True while the once-per-device setup guarded by `done` has not run on dev.
inline bool needs_setup(const std::atomic<bool>* done, int dev) {
  return device_slot(dev) && !done[dev].load(std::memory_order_acquire);
}
inline void mark_setup(std::atomic<bool>* done, int dev) {
  done[dev].store(true, std::memory_order_release);
}

// ------------------------------------------------------------- device status
// The sticky status word lives in status.cu; kernels receive its address as an
// argument and record the first error with atomicCAS (never trap).
__device__ __forceinline__ void record_error(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Returns the device address of the status word of the current device.
int* status_word();

// ----------------------------------------------------------------- numbers
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// Router logits follow one fixed fp32 order: the input index is cut into
// blocks of kRouteBlock consecutive elements; each block's partial sum is an
// ascending chain of fused multiply-adds from +0, and the logit is +0 plus
// the block sums in ascending block order (then + bias).
constexpr int kRouteBlock = 128;

// (c0, c1) = (b0 * a + c0, b1 * a + c1), each a single-rounding fp32 fma:
// the packed instruction gives the same results as two __fmaf_rn with half
// the instructions to issue.
__device__ __forceinline__ void fma2_rn(float& c0, float& c1, float b0, float b1, float a) {
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %2};\n\t"
      "mov.b64 rb, {%3, %4};\n\t"
      "mov.b64 rc, {%0, %1};\n\t"
      "fma.rn.f32x2 rc, rb, ra, rc;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "f"(a), "f"(b0), "f"(b1));
}

// The two largest of zr[0..n) (n >= 2, n <= NR) in the order of the
// slot-by-slot top-k selection: larger first, ties to the lower index, and a
// NaN kept only where that selection would keep it (a NaN first entry, or a
// NaN second entry when nothing later compares larger).  One pass.
template <int NR>
__device__ __forceinline__ void top2_of(const float* zr, int n, int& b0, float& z0, int& b1,
                                        float& z1) {
  b0 = 0;
  z0 = zr[0];
  b1 = -1;
  z1 = 0.0f;
#pragma unroll
  for (int i = 1; i < NR; ++i) {
    if (i < n) {
      if (zr[i] > z0) {
        b1 = b0;
        z1 = z0;
        b0 = i;
        z0 = zr[i];
      } else if (b1 < 0 || zr[i] > z1) {
        b1 = i;
        z1 = zr[i];
      }
    }
  }
}

// Load 8 consecutive elements (16 B for 16-bit types, 32 B for fp32) as fp32.
__device__ __forceinline__ void load8(const float* p, float* o) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* o) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const __half* p, float* o) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
    float2 f = __half22float2(h);
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// Gated activations of the bf16 tensor-core epilogues, whose result is rounded
// to bf16 (8 significant bits): the hardware exp2/reciprocal/tanh
// approximations (about 2^-21, 2^-22 and 2^-11 relative error) stay well
// below that rounding.  ACT is a compile-time constant so a SwiGLU kernel
// carries no trace of the capped variant.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <int ACT>
__device__ __forceinline__ float gated_act(float g, float v, float bg, float bu) {
  if (ACT == MOE_ACT_SITU_GLU) {  // beta * tanh(x / beta) soft caps
    g = bg * tanh_approx(__fdividef(g, bg));
    v = bu * tanh_approx(__fdividef(v, bu));
  }
  return __fdividef(g, 1.0f + __expf(-g)) * v;
}

// Four fp32 values to four OCP E4M3 codes (round to nearest even, magnitudes
// above 448 saturate to 448), v[0] in the lowest byte.
__device__ __forceinline__ uint32_t e4m3x4_rn(const float* v) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[0], v[1]), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(v[2], v[3]), __NV_SATFINITE, __NV_E4M3);
  return (lo & 0xFFFFu) | (hi << 16);
}

// ------------------------------------------- programmatic dependent launch
// Every kernel is launched with programmatic stream serialization: its CTAs
// may be scheduled while the previous kernel on the stream drains, and they
// wait in pdl_wait() (before their first global-memory access) until that
// kernel has finished and its writes are visible.  pdl_allow_next() lets the
// following kernel be scheduled early in turn.  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_allow_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------- host checks
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool valid_act_dtype(int32_t dt) {
  return dt == MOE_F32 || dt == MOE_BF16 || dt == MOE_F16;
}

inline size_t dtype_bytes(int32_t dt) { return dt == MOE_F32 ? 4 : 2; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Basic shape validity shared by every entry point.
inline bool shape_ok(const moe_shape* s) {
  if (!s) return false;
  if (s->T < 0 || s->d <= 0 || s->N <= 0 || s->N > 1024 || s->k <= 0 || s->k > 32) return false;
  if (s->k > s->N || (s->d % 8) != 0 || s->capacity < 0) return false;
  if ((int64_t)s->T * s->k >= (int64_t)1 << 31) return false;
  return true;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Launch errors reported by cudaLaunchKernelEx (launch_pdl) on this thread.
inline cudaError_t& pdl_launch_error() {
  static thread_local cudaError_t e = cudaSuccess;
  return e;
}

inline int launch_status() {
  const cudaError_t e = cudaGetLastError();
  const cudaError_t p = pdl_launch_error();
  pdl_launch_error() = cudaSuccess;
  return (e == cudaSuccess && p == cudaSuccess) ? MOE_OK : MOE_ERR_CUDA;
}

// Every kernel of the library asks for the maximum shared-memory carve-out, so
// consecutive launches on an SM never need a different L1/shared split (the
// tensor-core kernels need ~215 KB of shared memory).  Once per device and
// call site.
#define MOE_PREFER_SHARED(kernel)                                                      \
  do {                                                                                 \
    static std::atomic<bool> moe_done_[::moe::kMaxDevices];                            \
    int moe_dev_ = 0;                                                                  \
    if (cudaGetDevice(&moe_dev_) == cudaSuccess && ::moe::needs_setup(moe_done_, moe_dev_)) { \
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,     \
                           (int)cudaSharedmemCarveoutMaxShared);                       \
      ::moe::mark_setup(moe_done_, moe_dev_);                                          \
    }                                                                                  \
  } while (0)

// Launches kernel<<<grid, block, smem, st>>>(args...) with programmatic
// stream serialization (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) pdl_launch_error() = e;
  return e;
}

// Carves sub-buffers out of a caller workspace (256-byte aligned pieces).
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
  size_t used() const { return align_up(off, 256); }
};

// ------------------------------------------------------- internal launchers
// (defined in the per-step .cu files; all asynchronous on `st`)
size_t route_ws_bytes(const moe_shape& s);
// hist (optional, N <= 16 only): per router block of route_tokens_per_block(N)
// tokens, the count of its dispatches to each expert, [blocks][N].
int launch_route(const moe_shape& s, const void* u, int32_t u_dtype, const float* w_route,
                 const float* bias, int32_t* top_idx, float* top_w, float* probs, float* logits,
                 void* ws, cudaStream_t st, int32_t* hist = nullptr);
int route_tokens_per_block(int N);
// Permutation in one launch from the router's per-block counts (few experts;
// dispatch_small_ok says when): see dispatch_small in permute.cu.
bool dispatch_small_ok(const moe_shape& s);
// row_w (nullable): row_w[r] = top_w of the dispatch that owns grouped row r,
// for the down GEMM's weighted epilogue (also for launch_permute and
// launch_route_dispatch).
int launch_dispatch_small(const moe_shape& s, const int32_t* top_idx, const int32_t* hist,
                          int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* row_of,
                          int32_t* overflow, int32_t* totals, cudaStream_t st,
                          const float* top_w = nullptr, float* row_w = nullptr);
// Router + permutation + gather in one cooperative launch (route_dispatch.cu),
// for few experts when a CTA's token rows and the router rows fit on chip.
bool route_dispatch_ok(const moe_shape& s, int32_t dtype);
size_t route_dispatch_ws_bytes(const moe_shape& s);
int launch_route_dispatch(const moe_shape& s, const void* u, int32_t dtype, const float* w_route,
                          const float* bias, int32_t* top_idx, float* top_w, float* probs,
                          float* logits, int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                          int32_t* row_of, int32_t* overflow, int32_t* totals, void* x_rows,
                          void* ws, cudaStream_t st, float* row_w = nullptr);
size_t aux_stats_ws_bytes(int32_t N);
int launch_aux_stats(int32_t T, int32_t N, int32_t k, const float* probs, const int32_t* top_idx,
                     float* f, float* P, float* n_sum_fP, int32_t* loads, void* ws,
                     cudaStream_t st);
size_t permute_ws_bytes(const moe_shape& s);
int launch_permute(const moe_shape& s, const int32_t* top_idx, int32_t* counts, int32_t* offsets,
                   int32_t* perm_tok, int32_t* row_of, int32_t* overflow, int32_t* totals,
                   void* ws, cudaStream_t st, const float* top_w = nullptr,
                   float* row_w = nullptr);
int launch_gather(const moe_shape& s, int32_t width, const void* u, int32_t dtype,
                  const int32_t* perm_tok, const int32_t* offsets, void* x_rows, cudaStream_t st);
int launch_combine(const moe_shape& s, int32_t width, const float* y_rows, const int32_t* row_of,
                   const float* top_w, void* y, int32_t y_dtype, cudaStream_t st);
// y[t] = sum over kept slots s (ascending) of rows[row_of[t][s]], fp32 rows
// already weighted by their combine weights; fp32 sum, one rounding to y_dtype.
int launch_combine_weighted(const moe_shape& s, int32_t width, const float* rows,
                            const int32_t* row_of, void* y, int32_t y_dtype, cudaStream_t st);
size_t ffn_simt_ws_bytes(const moe_shape& s);
int launch_ffn_simt(const moe_shape& s, int32_t width, const float* x_rows, const int32_t* offsets,
                    const float* w_gate, const float* w_up, const float* w_down,
                    const moe_act& act, float* y_rows, void* ws, cudaStream_t st);
size_t ffn_tc_ws_bytes(const moe_shape& s, int32_t width);
// y_rows: fp32 expert outputs F(u) per grouped row, or (row_w != nullptr) the
// rows already weighted, row_w[r] * F(u) (the combine then only adds them).
int launch_ffn_tc(const moe_shape& s, int32_t width, const __nv_bfloat16* x_rows,
                  const int32_t* offsets, const __nv_bfloat16* w_gate, const __nv_bfloat16* w_up,
                  const __nv_bfloat16* w_down, const moe_act& act, void* y_rows, void* ws,
                  cudaStream_t st, const float* row_w = nullptr);

// Gather of the expert path fused with per-token E4M3 quantisation (fp8.cu):
// codes[r] = e4m3 codes of x[perm_tok[r]] / scales[r], rows r < offsets[N].
int launch_quant_gather_e4m3(const moe_shape& s, int cols, const __nv_bfloat16* x,
                             const int32_t* perm_tok, const int32_t* offsets, uint8_t* codes,
                             float* scales, cudaStream_t st);

// Fused single-launch expert FFN for small hidden widths (ffn_fused.cu).
bool ffn_fused_ok(int width, int h, int G);
int launch_ffn_fused(int G, int64_t R, int width, int h, const __nv_bfloat16* x_rows,
                     const int32_t* offsets, const __nv_bfloat16* w_gate,
                     const __nv_bfloat16* w_up, const __nv_bfloat16* w_down, const moe_act& act,
                     void* y_rows, cudaStream_t st, const float* row_w = nullptr);

// Grouped tcgen05 GEMM helpers (gemm_tc.cu).
enum TcMode { MODE_GATEUP = 0, MODE_STORE_F32 = 1, MODE_STORE_BF16 = 2 };

// One K-segment of a store-mode GEMM: A rows (weights) and B rows (tokens).
struct TcSeg {
  const void* a;      // [a_rows][K] bf16
  int64_t a_rows;
  int K;              // multiple of 64
  int arow;           // row offset into A added to the group's base row
  const void* b;      // [b_rows][b_cols] bf16
  int64_t b_rows;
  int b_cols;
  int bcol;           // column offset into B
};

// E4M3 operands of a grouped GEMM: codes in the operand arrays, fp32 scales
// per row of A (gate/up: gate rows, up rows) and per row of B (nullable: 1).
struct TcF8 {
  const float* a_scale[2];
  const float* b_scale;
};

// Gate/up GEMM with the fused activation: for group g and its rows of X,
// out[row][g * out_col_group + j] = act(X W_gate[g]^T, X W_up[g]^T)[j] as bf16
// (f8 == nullptr: bf16 X and weights), or as E4M3 codes with no scale (f8:
// E4M3 X and weights with their row scales; K a multiple of 128).
// offsets == nullptr: every group uses rows [0, T) of X.
int tc_gateup(const int32_t* offsets, int T, int G, const void* X, int64_t x_rows, int K,
              const void* w_gate, const void* w_up, int hidden, const moe_act& act, void* out,
              int out_ld, int out_col_group, cudaStream_t st, const TcF8* f8 = nullptr);
// Store-mode GEMM over 1..3 K-segments accumulated into one fp32 tile:
// out[row][g * m_rows + m] = sum_s A_s[g * a_rows + arow_s + m] . B_s[row][bcol_s ...].
// f8: one segment of E4M3 operands, fp32 output scaled by the row scales.
// b_row_scale (nullable): a factor per token row, applied to the fp32 result
// before the store (the combine weights of the grouped rows); with f8, its
// b_scale plays this part.
int tc_store(const int32_t* offsets, int T, int G, int m_rows, const TcSeg* segs, int nseg,
             void* out, int mode, int out_ld, cudaStream_t st, const TcF8* f8 = nullptr,
             const float* b_row_scale = nullptr);

}  // namespace moe
