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

// Programmatic dependent launch.  Every kernel is launched with the
// programmatic-stream-serialization attribute (unless FP8Q_PDL=0), so it may
// start while the previous kernel of its stream is still finishing.  It runs
// its prologue (barrier init, TMEM allocation, descriptor prefetch, and for
// the GEMMs an L2 prefetch of the first weight tiles: a cache hint with no
// visible effect, the tiles are loaded again after the wait), then
// griddep_wait() blocks until every earlier kernel of the stream has
// completed and its writes are visible.  Nothing before the wait reads or
// writes memory an earlier kernel may write.  griddep_launch_dependents()
// lets the next kernel begin its own prologue.  Launched without the
// attribute, both instructions do nothing.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Host-side helpers shared by the entry points.
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline fp8q_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

int num_sms();  // SM count of the current device (cached per device)

bool pdl_enabled();  // false when the environment sets FP8Q_PDL=0 (read once)

// Launch `kern` on `stream` with programmatic dependent launch (when enabled)
// and, for cluster_x > 1, clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline fp8q_status launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, unsigned cluster_x, Args&&... args) {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...) != cudaSuccess) return FP8Q_ERR_CUDA;
  return launch_status();
}

}  // namespace fp8q
