// fp8q_quant.cu -- dynamic FP8 activation quantization fused with its producer.
//
// Ops ("Helion in vLLM" (24-ai.news), section "Kernels integrated into vLLM"):
//   items 1, 5  per-token / per-1x128-group quant          -> fp8q_group_quant
//   items 2, 6  RMSNorm + per-token / per-block quant       -> fp8q_rmsnorm_quant
//   items 3, 7  SiLU*mul + per-token / per-block quant      -> fp8q_silu_mul_quant
//
// One CTA owns one row.  Every thread loads its 16-byte chunks of the row
// (8 bf16 each; chunk c of the row goes to thread c mod T, so a warp reads 512
// contiguous bytes per load), all loads issued before any arithmetic.  The row
// then stays in registers as packed bf16 y values: one HBM read, one write of
// the codes.  Group amax = shuffle over the 16 threads that own one 128-wide
// group; row amax and the RMSNorm sum of squares = warp shuffle + a shared-
// memory pass over the warps.
//
// Exactness.  Codes and scales are meant to equal the definition bit for bit:
//   - the scale is an IEEE fp32 division, the codes come from an IEEE fp32
//     division x/s and the hardware saturating RNE e4m3 conversion;
//   - y must be the correctly rounded bf16 of the op's real value.  The fast
//     path computes it in fp32 with a known error bound (a few fp32 ulps); when
//     that fp32 value lies within the bound of a bf16 rounding midpoint, or is
//     tiny, the element is recomputed in fp64 and rounded to bf16 once
//     (round-to-odd to fp32, then nearest-even to bf16).  The RMSNorm sum of
//     squares and 1/sqrt are fp64.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp8q_common.cuh"

namespace fp8q {
namespace {

enum { OP_PLAIN = 0, OP_RMS = 1, OP_SILU = 2 };
constexpr int kMaxThreads = 512;  // rows up to 8 * 8 * 512 = 32768 elements

struct QuantParams {
  const uint16_t* x;   // bf16 bits
  const uint16_t* w;   // bf16 bits (RMSNorm weight) or null
  float eps;
  int64_t M, L, ldx;   // L = row length of y (K, H or I)
  int group;           // 128 or L
  int ue8m0;
  uint8_t* q;
  int64_t ldq;
  float* s;
  int64_t s_sm, s_sg;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_bits_rn(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// Round an fp64 value to bf16 with a single rounding: round-to-odd to fp32
// (24 bits, >= 2 more than bf16's 8, so the later rounding is exact), then
// nearest-even to bf16.
__device__ __noinline__ uint32_t f64_to_bf16_bits_rn(double v) {
  float f = __double2float_rz(v);
  if (static_cast<double>(f) != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f32_to_bf16_bits_rn(f);
}

// True when the fp32 value p may round to a different bf16 than a real value
// within `margin` fp32 ulps of it: p lies within margin ulps of a rounding
// midpoint (low 16 bits 0x8000), or p is tiny (where fp32 loses precision).
__device__ __forceinline__ bool bf16_rounding_unsafe(float p, int margin) {
  const uint32_t u = __float_as_uint(p);
  const int d = static_cast<int>(u & 0xFFFFu) - 0x8000;
  const bool tiny = (u & 0x7FFFFFFFu) != 0u && (u & 0x7F800000u) < 0x0D800000u;  // |p| < 2^-100
  return (d <= margin && d >= -margin) || tiny;
}

// RMSNorm element: bf16(bf16(x * r) * w).  Fast path error: r32 = fl(r) and
// x*r32 each add <= 2^-24 relative, so |p - x r| <= 2 ulps; margin 8.
__device__ __forceinline__ uint32_t rms_elem(float x, float r32, double r, float w) {
  const float p = __fmul_rn(x, r32);
  uint32_t nb;
  if (bf16_rounding_unsafe(p, 8)) nb = f64_to_bf16_bits_rn(static_cast<double>(x) * r);
  else nb = f32_to_bf16_bits_rn(p);
  // n * w is exact in fp32 (8-bit x 8-bit significands): one rounding to bf16.
  return f32_to_bf16_bits_rn(__fmul_rn(bf16_bits_to_f32(nb), w));
}

// SiLU*mul element: bf16(silu(g) * u), silu(g) = g / (1 + e^-g).  Fast path
// error: expf <= 2 ulp, then three IEEE roundings: |p - silu(g) u| <= 7 ulps;
// margin 16.  Gates below -85 make e^-g overflow fp32: always the fp64 path.
__device__ __forceinline__ uint32_t silu_mul_elem(float g, float u) {
  const float e = expf(-g);
  const float sl = __fdiv_rn(g, __fadd_rn(1.0f, e));
  const float p = __fmul_rn(sl, u);
  if (g < -85.0f || bf16_rounding_unsafe(p, 16)) {
    const double gd = static_cast<double>(g);
    return f64_to_bf16_bits_rn(gd / (1.0 + exp(-gd)) * static_cast<double>(u));
  }
  return f32_to_bf16_bits_rn(p);
}

__device__ __forceinline__ float group_scale(float amax, int ue8m0) {
  float s = __fdiv_rn(fmaxf(amax, 1e-10f), 448.0f);
  if (ue8m0) {
    uint32_t u = __float_as_uint(s);          // s >= 2.2e-13: a positive normal
    if (u & 0x007FFFFFu) u = (u & 0xFF800000u) + 0x00800000u;
    s = __uint_as_float(u);
  }
  return s;
}

// 8 bf16 values (one chunk) -> 8 e4m3 codes, y / s with IEEE division.
__device__ __forceinline__ uint2 quantize_chunk(const uint4& y, float s) {
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t v = w[2 * h + j];
      float2 t;
      t.x = __fdiv_rn(bf16_bits_to_f32(v & 0xFFFFu), s);
      t.y = __fdiv_rn(bf16_bits_to_f32(v >> 16), s);
      const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(t, __NV_SATFINITE, __NV_E4M3);
      packed |= static_cast<uint32_t>(c) << (16 * j);
    }
    out[h] = packed;
  }
  return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ float chunk_amax(const uint4& y) {
  // |bf16| max on the bit patterns: clear the sign, compare as integers.
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = max(m, w[i] & 0x7FFFu);
    m = max(m, (w[i] >> 16) & 0x7FFFu);
  }
  return bf16_bits_to_f32(m);
}

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename T, typename Op>
__device__ __forceinline__ T block_reduce(T v, Op op, T* smem) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();  // smem may still be read by a previous reduction
  if (lane == 0) smem[warp] = v;
  __syncthreads();
  v = smem[0];
  for (int i = 1; i < nw; ++i) v = op(v, smem[i]);
  return v;
}

struct MaxOp { __device__ float operator()(float a, float b) const { return fmaxf(a, b); } };
struct SumOp { __device__ double operator()(double a, double b) const { return a + b; } };

template <int OP, bool PER_TOKEN, int CH>
__global__ void __launch_bounds__(kMaxThreads, 1) quant_rows_kernel(const QuantParams p) {
  __shared__ double red_d[32];
  __shared__ float red_f[32];
  const int T = blockDim.x, tid = threadIdx.x;
  const int64_t nchunks = p.L >> 3;

  for (int64_t row = blockIdx.x; row < p.M; row += gridDim.x) {
    const uint16_t* xr = p.x + row * p.ldx;
    uint4 y[CH];
    bool valid[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) valid[i] = (tid + static_cast<int64_t>(i) * T) < nchunks;

    if constexpr (OP == OP_PLAIN) {
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if (valid[i]) y[i] = ld_stream(xr + (tid + static_cast<int64_t>(i) * T) * 8);
    } else if constexpr (OP == OP_SILU) {
      // gate and up chunks are loaded in batches of 4 chunks to bound registers.
#pragma unroll
      for (int i0 = 0; i0 < CH; i0 += 4) {
        uint4 g[4], u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (valid[i0 + i]) {
            const int64_t off = (tid + static_cast<int64_t>(i0 + i) * T) * 8;
            g[i] = ld_stream(xr + off);
            u[i] = ld_stream(xr + p.L + off);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (valid[i0 + i]) {
            const uint32_t gw[4] = {g[i].x, g[i].y, g[i].z, g[i].w};
            const uint32_t uw[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t lo = silu_mul_elem(bf16_bits_to_f32(gw[j] & 0xFFFFu),
                                                bf16_bits_to_f32(uw[j] & 0xFFFFu));
              const uint32_t hi = silu_mul_elem(bf16_bits_to_f32(gw[j] >> 16),
                                                bf16_bits_to_f32(uw[j] >> 16));
              o[j] = lo | (hi << 16);
            }
            y[i0 + i] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    } else {  // OP_RMS
      uint4 xv[CH];
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if (valid[i]) xv[i] = ld_stream(xr + (tid + static_cast<int64_t>(i) * T) * 8);
      double ss = 0.0;
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if (valid[i]) {
          const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const double a = bf16_bits_to_f32(xw[j] & 0xFFFFu);
            const double b = bf16_bits_to_f32(xw[j] >> 16);
            ss = fma(a, a, ss);
            ss = fma(b, b, ss);
          }
        }
      }
      ss = block_reduce(ss, SumOp(), red_d);
      const double r = 1.0 / sqrt(ss / static_cast<double>(p.L) + static_cast<double>(p.eps));
      const float r32 = static_cast<float>(r);
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if (valid[i]) {
          const uint4 wv = *reinterpret_cast<const uint4*>(p.w + (tid + static_cast<int64_t>(i) * T) * 8);
          const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
          const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t lo = rms_elem(bf16_bits_to_f32(xw[j] & 0xFFFFu), r32, r,
                                         bf16_bits_to_f32(ww[j] & 0xFFFFu));
            const uint32_t hi = rms_elem(bf16_bits_to_f32(xw[j] >> 16), r32, r,
                                         bf16_bits_to_f32(ww[j] >> 16));
            o[j] = lo | (hi << 16);
          }
          y[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }

    uint8_t* qr = p.q + row * p.ldq;
    if constexpr (PER_TOKEN) {
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if (valid[i]) amax = fmaxf(amax, chunk_amax(y[i]));
      amax = block_reduce(amax, MaxOp(), red_f);
      const float s = group_scale(amax, p.ue8m0);
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if (valid[i]) {
          const int64_t c = tid + static_cast<int64_t>(i) * T;
          *reinterpret_cast<uint2*>(qr + c * 8) = quantize_chunk(y[i], s);
        }
      }
      if (tid == 0) p.s[row * p.s_sm] = s;
    } else {
      // 128-wide groups: the 16 threads tid & ~15 .. +15 own one group per i
      // (T is a multiple of 32 and L of 128, so whole half-warps are valid or not).
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        float a = valid[i] ? chunk_amax(y[i]) : 0.0f;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        if (valid[i]) {
          const int64_t c = tid + static_cast<int64_t>(i) * T;
          const float s = group_scale(a, p.ue8m0);
          *reinterpret_cast<uint2*>(qr + c * 8) = quantize_chunk(y[i], s);
          if ((tid & 15) == 0) p.s[row * p.s_sm + (c >> 4) * p.s_sg] = s;
        }
      }
    }
  }
}

// Threads per row: enough that CH chunks per thread cover the row; a multiple
// of 32 (whole warps), at least 32.
inline int threads_for(int64_t nchunks, int ch) {
  int64_t t = (nchunks + ch - 1) / ch;
  t = ((t + 31) / 32) * 32;
  return static_cast<int>(t < 32 ? 32 : t);
}

template <int OP>
fp8q_status launch_quant(const QuantParams& p, cudaStream_t stream) {
  if (p.M == 0) return FP8Q_OK;
  const int64_t nchunks = p.L / 8;
  const bool per_token = p.group == p.L;
  const int ch = nchunks > 512 ? 8 : 4;
  const int T = threads_for(nchunks, ch);
  if (T > kMaxThreads) return FP8Q_ERR_UNSUPPORTED;
  const int64_t grid = p.M < (1LL << 30) ? p.M : (1LL << 30);
  const dim3 g(static_cast<unsigned>(grid)), b(T);
  if (ch == 8) {
    if (per_token) quant_rows_kernel<OP, true, 8><<<g, b, 0, stream>>>(p);
    else quant_rows_kernel<OP, false, 8><<<g, b, 0, stream>>>(p);
  } else {
    if (per_token) quant_rows_kernel<OP, true, 4><<<g, b, 0, stream>>>(p);
    else quant_rows_kernel<OP, false, 4><<<g, b, 0, stream>>>(p);
  }
  return launch_status();
}

// Host-side validation shared by the three ops (row length L of y).
fp8q_status check_common(const void* x, int64_t M, int64_t L, int64_t ldx, int64_t ld_in_min,
                         int group, int ue8m0, const void* q, int64_t ldq, const float* s,
                         int64_t s_sm, int64_t s_sg) {
  if (M < 0 || L <= 0 || L % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (ldx < ld_in_min || ldx % 8 != 0 || ldq < L || ldq % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (!(group == 128 && L % 128 == 0) && static_cast<int64_t>(group) != L) return FP8Q_ERR_INVALID_ARG;
  if (ue8m0 != 0 && ue8m0 != 1) return FP8Q_ERR_INVALID_ARG;
  if (s_sm < 0 || s_sg < 0) return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;  // nothing is read or written: pointers may be null
  if (!x || !q || !s) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, 4)) return FP8Q_ERR_INVALID_ARG;
  return FP8Q_OK;
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_group_quant(const void* x, int64_t M, int64_t K, int64_t ldx,
                                        int group_size, int ue8m0, void* q, int64_t ldq,
                                        float* scales, int64_t s_stride_m, int64_t s_stride_g,
                                        void* stream) {
  fp8q_status st = check_common(x, M, K, ldx, K, group_size, ue8m0, q, ldq, scales, s_stride_m,
                                s_stride_g);
  if (st != FP8Q_OK) return st;
  QuantParams p{static_cast<const uint16_t*>(x), nullptr, 0.0f, M, K, ldx, group_size, ue8m0,
                static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g};
  return launch_quant<OP_PLAIN>(p, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_rmsnorm_quant(const void* x, const void* w, float eps, int64_t M,
                                          int64_t H, int64_t ldx, int group_size, int ue8m0,
                                          void* q, int64_t ldq, float* scales,
                                          int64_t s_stride_m, int64_t s_stride_g, void* stream) {
  fp8q_status st = check_common(x, M, H, ldx, H, group_size, ue8m0, q, ldq, scales, s_stride_m,
                                s_stride_g);
  if (st != FP8Q_OK) return st;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return FP8Q_ERR_INVALID_ARG;
  if (M > 0 && (!w || !aligned(w, 16))) return FP8Q_ERR_INVALID_ARG;
  QuantParams p{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w), eps, M, H, ldx,
                group_size, ue8m0, static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g};
  return launch_quant<OP_RMS>(p, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_silu_mul_quant(const void* x, int64_t M, int64_t I, int64_t ldx,
                                           int group_size, int ue8m0, void* q, int64_t ldq,
                                           float* scales, int64_t s_stride_m, int64_t s_stride_g,
                                           void* stream) {
  if (I > (INT64_MAX / 4)) return FP8Q_ERR_INVALID_ARG;
  fp8q_status st = check_common(x, M, I, ldx, 2 * I, group_size, ue8m0, q, ldq, scales,
                                s_stride_m, s_stride_g);
  if (st != FP8Q_OK) return st;
  QuantParams p{static_cast<const uint16_t*>(x), nullptr, 0.0f, M, I, ldx, group_size, ue8m0,
                static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g};
  return launch_quant<OP_SILU>(p, static_cast<cudaStream_t>(stream));
}
