// Exhaustive worst-case relative error, on this GPU, of the hardware
// approximations the quant kernels' fast paths rely on (their rounding
// brackets are sized from these bounds): ex2.approx.ftz.f32 on [-126, 128),
// rcp.approx.ftz.f32 on every mantissa of several binades, and the
// ex2-based e^x (same construction as exp_fast in fp8q_quant.cu) on
// [-87, 87], rsqrtf (the RMSNorm fast path) on [1, 4), and the
// Newton-refined reciprocal of the SiLU fast path.  References in fp64.
// Prints five relative errors.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <cuda_runtime.h>

__device__ unsigned int g_max[5];

__device__ __forceinline__ float ex2a(float a) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}
__device__ __forceinline__ float rcpa(float a) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}
__device__ __forceinline__ float exp_fast(float x) {
  const float L2E = 1.44269502f, L2E_LO = 1.925963e-8f;
  const float a = __fmul_rn(x, L2E);
  const float lo = __fmaf_rn(x, L2E_LO, __fmaf_rn(x, L2E, -a));
  const float e = ex2a(a);
  return __fmaf_rn(e, __fmul_rn(lo, 0.693147182f), e);
}
__device__ __forceinline__ void upd(int k, double rel) {
  atomicMax(&g_max[k], __float_as_uint(static_cast<float>(fabs(rel))));
}
__global__ void k_ex2(uint32_t n, uint32_t sign) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float x = __uint_as_float(i | sign);
    if (!(x >= -126.0f && x < 128.0f)) continue;
    const double ref = exp2(static_cast<double>(x));
    upd(0, (static_cast<double>(ex2a(x)) - ref) / ref);
  }
}
__global__ void k_exp(uint32_t n, uint32_t sign) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float x = __uint_as_float(i | sign);
    if (!(x >= -87.0f && x <= 87.0f)) continue;
    const double ref = exp(static_cast<double>(x));
    upd(2, (static_cast<double>(exp_fast(x)) - ref) / ref);
  }
}
__global__ void k_rcp(int e) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (1u << 23); i += gridDim.x * blockDim.x) {
    const float x = __uint_as_float((static_cast<uint32_t>(e + 127) << 23) | i);
    const double ref = 1.0 / static_cast<double>(x);
    upd(1, (static_cast<double>(rcpa(x)) - ref) / ref);
  }
}
// 1/d by rcp.approx of -d and one Newton step (the SiLU fast path's
// reciprocal, d = 1 + e^-g >= 1), every mantissa of several binades.
__global__ void k_rcp_newton(int e) {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (1u << 23); i += gridDim.x * blockDim.x) {
    const float d = __uint_as_float((static_cast<uint32_t>(e + 127) << 23) | i);
    const float nr0 = rcpa(-d);
    const float h = __fmaf_rn(d, nr0, 1.0f);
    const float r1 = -__fmaf_rn(nr0, h, nr0);
    const double ref = 1.0 / static_cast<double>(d);
    upd(4, (static_cast<double>(r1) - ref) / ref);
  }
}
// rsqrtf on every fp32 of [1, 4) (both exponent parities; relative error is
// the same in every other binade of normal numbers).
__global__ void k_rsqrt() {
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < (1u << 24); i += gridDim.x * blockDim.x) {
    const float x = __uint_as_float(0x3F800000u + i);
    const double ref = 1.0 / sqrt(static_cast<double>(x));
    upd(3, (static_cast<double>(rsqrtf(x)) - ref) / ref);
  }
}
int main() {
  const unsigned int z[5] = {0, 0, 0, 0, 0};
  cudaMemcpyToSymbol(g_max, z, sizeof(z));
  for (uint32_t sign : {0u, 0x80000000u}) {
    k_ex2<<<148 * 8, 256>>>(0x43000000u, sign);
    k_exp<<<148 * 8, 256>>>(0x42AE0000u, sign);
  }
  for (int e : {-120, -60, -10, -1, 0, 1, 10, 60, 120}) k_rcp<<<148 * 8, 256>>>(e);
  k_rsqrt<<<148 * 8, 256>>>();
  for (int e : {0, 1, 10, 60, 120}) k_rcp_newton<<<148 * 8, 256>>>(e);
  if (cudaDeviceSynchronize() != cudaSuccess) return 1;
  unsigned int m[5];
  cudaMemcpyFromSymbol(m, g_max, sizeof(m));
  float f[5];
  for (int i = 0; i < 5; ++i) std::memcpy(&f[i], &m[i], 4);
  std::printf("%.9e %.9e %.9e %.9e %.9e\n", f[0], f[1], f[2], f[3], f[4]);
  return 0;
}
