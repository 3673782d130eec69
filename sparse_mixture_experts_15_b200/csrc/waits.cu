// Checks of the library's bounded device waits: each kernel here runs one of
// the waits the persistent kernels use (the grid barrier of the cooperative
// kernels, the mbarrier wait of the tcgen05 kernels) on a condition that
// nothing ever satisfies, with a short budget.  The wait gives up, records
// MOE_ERR_TIMEOUT in the status word and the kernel returns normally, so the
// CUDA context stays usable.  Nothing faults, traps or spins without a bound.
#include "common.cuh"
#include "grid_sync.cuh"
#include "tc_primitives.cuh"

namespace moe {
namespace {

// Arrival counter and abort word of the grid-barrier check; zeroed before
// every launch.  Every call shares them (calls that overlap on the GPU race).
__device__ unsigned g_wait_check_bar[2];

// Every CTA arrives once; the barrier waits for one arrival more than the
// launch has CTAs, which nothing adds.
__global__ void wait_check_grid(unsigned* bar, unsigned long long budget_ns, int* status) {
  grid_arrive(bar);
  grid_wait(bar, gridDim.x + 1u, status, budget_ns);
}

// A fresh mbarrier whose phase 0 never completes (its one expected arrival
// never comes); the same bounded wait the tcgen05 producer / MMA / epilogue
// roles use.
__global__ void wait_check_mbar(long long budget_cycles, int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(&bar), 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !tc::mbar_wait(tc::smem_u32(&bar), 0u, nullptr, budget_cycles))
    record_error(status, MOE_ERR_TIMEOUT);
  __syncthreads();
}

}  // namespace
}  // namespace moe

extern "C" int moe_wait_check(int32_t kind, int64_t budget_ns, void* stream) {
  using namespace moe;
  if ((kind != MOE_WAIT_GRID_BARRIER && kind != MOE_WAIT_MBARRIER) || budget_ns < 1000 ||
      budget_ns > 2000000000LL)
    return MOE_ERR_INVALID_ARG;
  int* status = status_word();
  if (!status) return MOE_ERR_CUDA;
  cudaStream_t st = as_stream(stream);
  if (kind == MOE_WAIT_GRID_BARRIER) {
    void* bar = nullptr;
    if (cudaGetSymbolAddress(&bar, g_wait_check_bar) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(bar, 0, sizeof(g_wait_check_bar), st) != cudaSuccess) return MOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(32);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // both CTAs co-resident
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, wait_check_grid, static_cast<unsigned*>(bar),
                           (unsigned long long)budget_ns, status) != cudaSuccess)
      return MOE_ERR_CUDA;
  } else {
    // clock64 counts SM cycles: at 2 cycles per ns (about the B200's top SM
    // clock) the wait lasts about budget_ns; at lower clocks, longer.
    wait_check_mbar<<<1, 32, 0, st>>>((long long)budget_ns * 2, status);
  }
  return launch_status();
}
