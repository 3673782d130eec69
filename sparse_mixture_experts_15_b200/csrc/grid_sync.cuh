// Bounded grid-wide barrier of the cooperative (persistent) kernels: every
// CTA of the launch is co-resident, so a CTA may wait for all others.
#pragma once

#include "common.cuh"

namespace moe {

constexpr unsigned long long kBarrierBudgetNs = 2000000000ull;  // 2 s of device time

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Arrival counter bar[0] (zeroed before the launch) and abort flag bar[1].
// Barrier number n of the launch completes when bar[0] reaches G * (n + 1).
// grid_arrive: after the CTA's own work (bar.sync), thread 0 publishes it
// (fence.acq_rel at gpu scope, then a relaxed add).  The CTA may issue
// independent copies before grid_wait, which polls with acquire loads and
// returns false (every CTA then returns) on timeout or abort.
__device__ __forceinline__ void grid_arrive(unsigned* bar) {
  __syncthreads();
  if (threadIdx.x == 0)
    asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(bar)
                 : "memory");
}

static __device__ bool grid_wait(unsigned* bar, unsigned target, int* status,
                                 unsigned long long budget_ns = kBarrierBudgetNs) {
  __shared__ int ok;
  if (threadIdx.x == 0) {
    int good = 1;
    const unsigned long long t0 = global_ns();
    unsigned polls = 0;
    while (ld_acquire(bar) < target) {
      if ((++polls & 15u) == 0) {
        if (ld_acquire(bar + 1) != 0u) {
          good = 0;
          break;
        }
        if (global_ns() - t0 > budget_ns) {
          record_error(status, MOE_ERR_TIMEOUT);
          atomicExch(bar + 1, 1u);
          good = 0;
          break;
        }
      }
    }
    ok = good;
  }
  __syncthreads();
  return ok != 0;
}

}  // namespace moe
