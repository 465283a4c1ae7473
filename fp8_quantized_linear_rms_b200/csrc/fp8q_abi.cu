// fp8q_abi.cu -- status, version and device-query entry points of libfp8q.
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "fp8q_common.cuh"

namespace fp8q {

__device__ int g_device_status = 0;

// Per-device caches below are atomics: concurrent first calls may both fill
// an entry, with the same value.
int* device_status_ptr() {
  static std::atomic<int*> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  int* c = cache[dev].load(std::memory_order_relaxed);
  if (c == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    c = static_cast<int*>(p);
    cache[dev].store(c, std::memory_order_relaxed);
  }
  return c;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("FP8Q_PDL");
    return !(v && v[0] == '0' && v[1] == '\0');
  }();
  return on;
}

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace fp8q

extern "C" fp8q_status fp8q_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FP8Q_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, fp8q::g_device_status, sizeof(int)) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(fp8q::g_device_status, &zero, sizeof(int)) != cudaSuccess)
    return FP8Q_ERR_CUDA;
  return static_cast<fp8q_status>(v);
}

extern "C" const char* fp8q_status_string(fp8q_status s) {
  switch (s) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_INVALID_ARG: return "invalid argument";
    case FP8Q_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case FP8Q_ERR_CUDA: return "CUDA error";
    case FP8Q_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

extern "C" const char* fp8q_version(void) { return "fp8q 0.1 sm_100a"; }
