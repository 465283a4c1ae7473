// fp8q_common.cuh -- shared device helpers of libfp8q (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fp8q.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libfp8q is written for sm_100a (B200) only"
#endif

namespace fp8q {

// Device status word (one per device that loaded the library): kernels that
// give up on a wait record FP8Q_ERR_TIMEOUT there through the pointer the
// host passes them; fp8q_last_device_status reads and clears it.
int* device_status_ptr();  // device address of the status word (nullptr on error)

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Host-side helpers shared by the entry points.
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline fp8q_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int num_sms();  // SM count of the current device (cached per device)

}  // namespace fp8q
