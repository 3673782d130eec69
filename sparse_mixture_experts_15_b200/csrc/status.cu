// Sticky device status word, status strings and the capacity helper.
#include <cmath>

#include "common.cuh"

namespace moe {

__device__ int g_status_word = 0;

int* status_word() {
  // One address per device, looked up once with that device current.
  static std::atomic<int*> addr[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || !device_slot(dev)) return nullptr;
  int* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    a = static_cast<int*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace moe

extern "C" const char* moe_status_string(int32_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: bad pointer, size or alignment";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: combination not implemented";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA runtime call failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait ran out";
    case MOE_ERR_BOUNDS: return "MOE_ERR_BOUNDS: a device index was out of range";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace too small";
    default: return "unknown status";
  }
}

extern "C" int moe_device_status(void* stream, int32_t* status) {
  if (!status) return MOE_ERR_INVALID_ARG;
  int* w = moe::status_word();
  if (!w) return MOE_ERR_CUDA;
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, w, sizeof(int), cudaMemcpyDeviceToHost,
                                  moe::as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(moe::as_stream(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *status = v;
  return MOE_OK;
}

extern "C" int moe_reset_device_status(void* stream) {
  int* w = moe::status_word();
  if (!w) return MOE_ERR_CUDA;
  return moe::cuda_status(cudaMemsetAsync(w, 0, sizeof(int), moe::as_stream(stream)));
}

extern "C" int moe_capacity(int64_t T, int32_t N, int32_t k, double factor, int32_t* capacity) {
  if (!capacity || T < 0 || N <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (!(factor > 0.0)) {
    *capacity = 0;
    return MOE_OK;
  }
  double c = std::ceil(factor * (double)(k * T) / (double)N);
  if (c > 2147483647.0) return MOE_ERR_INVALID_ARG;
  *capacity = (int32_t)c;
  return MOE_OK;
}
