// fp8q_rope.cu -- fused_qk_norm_rope: per-head RMSNorm of the q and k heads of
// a packed qkv activation, then the rotary embedding at each token's position,
// in place ("Helion in vLLM" (24-ai.news), section "Kernels integrated into
// vLLM", item 4; the op's arguments as the vllm PR #44010 page lists them in
// section "Code analysis").
//
//   row t of qkv = [q heads (hq) | k heads (hk) | v heads (hv)], D bf16 each
//   q / k head:  r = 1/sqrt(mean(x^2) + eps), n = bf16(x r), y = bf16(n w)
//   rotary:      pairs (i, i + D/2) (NeoX) or (2i, 2i + 1) (GPT-J) with
//                cos = cache[p][i], sin = cache[p][D/2 + i], p = positions[t]:
//                a' = bf16(a cos - b sin), b' = bf16(b cos + a sin)
//
// HBM-bound: every q/k element is read and written once.  A head is owned by
// D/8 consecutive threads, 8 elements (16 bytes) each, so consecutive thread
// groups read consecutive heads of a token (coalesced); the group reduces the
// sum of squares with shuffles, exchanges NeoX partners with one shuffle
// (GPT-J pairs sit inside a thread) and each thread keeps several heads in
// flight.  The norm is exact, as in the quant kernels: the sum of squares in
// fp64 (squares of bf16 values are exact there), r = 1/sqrt(ss/D + eps) in
// fp64, and n = bf16(x r) from the two ends rz(x r_lo) and rz(x r_hi) + 1 ulp
// of fp32 values r_lo <= r <= r_hi; the rare elements whose ends round
// differently are rounded from fp64 once.  y = bf16(n w) is one exactly
// rounded bf16 product.  The rotation is fp32: a cos - b sin as
// fma(a, cos, -p) - e with p = fl(b sin) and e its exact FMA residual, so the
// difference keeps its accuracy when the two products nearly cancel; each
// output is rounded to bf16 once.
#include <cuda_bf16.h>

#include <atomic>

#include "fp8q_common.cuh"

namespace fp8q {
namespace {

struct RopeParams {
  uint16_t* qkv;               // bf16 bits, [T, ld]
  int64_t T, ld;
  int hq, hk;                  // q and k heads (v heads follow, untouched)
  float eps;
  const uint16_t* qw;          // [D] bf16
  const uint16_t* kw;          // [D] bf16
  const float* cs;             // [max_pos, D] fp32: cos (D/2) | sin (D/2)
  const int64_t* pos;          // [T]
  int64_t max_pos;
  int* status;                 // device status word (a position out of range)
};

constexpr int kRopeThreads = 256;
constexpr int kRopeItems = 4;  // heads per thread in flight

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// u v + s w (s = +-1) with the product w-term split exactly: p = fl(s w),
// e = the rounding error of p (an FMA residual), result fma(u, v, p) + e.
__device__ __forceinline__ float rot(float u, float v, float s, float w) {
  const float pr = s * w;
  const float e = fmaf(s, w, -pr);
  return fmaf(u, v, pr) + e;
}

// bf16 (nearest even) of a double with one rounding: round to odd at fp32
// (24 bits, two more than bf16 needs), then nearest-even to bf16.
__device__ __noinline__ uint32_t f64_to_bf16_rn(double v) {
  float f = __double2float_rz(v);
  if (static_cast<double>(f) != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// n = bf16(x r) exactly: the ends of |x r| from r_lo <= r <= r_hi decide the
// rounding when they agree; otherwise x r is rounded from fp64.
__device__ __forceinline__ uint32_t norm_bf16(float x, float r_lo, float r_hi, double r) {
  const uint32_t a = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rz(x, r_lo))));
  const uint32_t b = static_cast<uint32_t>(__bfloat16_as_ushort(
      __float2bfloat16_rn(__uint_as_float(__float_as_uint(__fmul_rz(x, r_hi)) + 1u))));
  return a == b ? a : f64_to_bf16_rn(static_cast<double>(x) * r);
}

__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {   // one rounding
  const __nv_bfloat162 y = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                   *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&y);
}

template <int D, bool NEOX>
__global__ void __launch_bounds__(kRopeThreads) qk_norm_rope_kernel(const RopeParams p) {
  constexpr int G = D / 8;                       // threads per head
  constexpr int GROUPS = kRopeThreads / G;       // heads per block per item slot
  const int g = threadIdx.x % G;                 // 16-byte chunk of the head
  const int grp = threadIdx.x / G;
  const int heads = p.hq + p.hk;
  const int64_t items = p.T * heads;

  griddep_wait();                                // qkv may come from the previous kernel
  griddep_launch_dependents();

  const uint4 wq = __ldg(reinterpret_cast<const uint4*>(p.qw) + g);
  const uint4 wk = __ldg(reinterpret_cast<const uint4*>(p.kw) + g);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * GROUPS * kRopeItems;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * GROUPS * kRopeItems; base < items;
       base += stride) {
    uint4 x[kRopeItems];
    int64_t t[kRopeItems];
    int h[kRopeItems];
    bool ok[kRopeItems];
#pragma unroll
    for (int u = 0; u < kRopeItems; ++u) {
      const int64_t it = base + grp + static_cast<int64_t>(u) * GROUPS;
      ok[u] = it < items;
      t[u] = ok[u] ? it / heads : 0;
      h[u] = ok[u] ? static_cast<int>(it - t[u] * heads) : 0;
      x[u] = ok[u] ? *reinterpret_cast<const uint4*>(p.qkv + t[u] * p.ld + h[u] * D + 8 * g)
                   : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kRopeItems; ++u) {
      const uint32_t xw[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
      double ss = 0.0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const double lo = bf_lo(xw[k]), hi = bf_hi(xw[k]);
        ss = __fma_rn(lo, lo, __fma_rn(hi, hi, ss));
      }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      const double r = 1.0 / sqrt(ss / static_cast<double>(D) + static_cast<double>(p.eps));
      const float r_lo = __double2float_rd(r * (1.0 - 0x1p-40));
      const float r_hi = __double2float_ru(r * (1.0 + 0x1p-40));
      const uint4 w = h[u] < p.hq ? wq : wk;
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      float y[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t nw = norm_bf16(bf_lo(xw[k]), r_lo, r_hi, r) |
                            (norm_bf16(bf_hi(xw[k]), r_lo, r_hi, r) << 16);
        const uint32_t yw = bf2_mul(nw, ww[k]);
        y[2 * k] = bf_lo(yw);
        y[2 * k + 1] = bf_hi(yw);
      }
      // cos / sin of this thread's pairs at the token's position
      int64_t ps = ok[u] ? __ldg(p.pos + t[u]) : 0;
      if (ps < 0 || ps >= p.max_pos) {         // out of range: flag it, use position 0
        if (ok[u]) record_status(p.status, FP8Q_ERR_INVALID_ARG);
        ps = 0;
      }
      const float* cs = p.cs + ps * D;
      float out[8];
      if constexpr (NEOX) {
        // partner thread g ^ G/2 holds the other half of every pair
        float z[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) z[j] = __shfl_xor_sync(0xFFFFFFFFu, y[j], G / 2);
        const int i0 = (8 * g) % (D / 2);
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(cs + i0));
        const float4 c1 = __ldg(reinterpret_cast<const float4*>(cs + i0 + 4));
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(cs + D / 2 + i0));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(cs + D / 2 + i0 + 4));
        const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        const bool first = g < G / 2;          // this thread holds the a's
#pragma unroll
        for (int j = 0; j < 8; ++j) out[j] = rot(y[j], c[j], first ? -z[j] : z[j], sn[j]);
      } else {
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(cs + 4 * g));
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(cs + D / 2 + 4 * g));
        const float c[4] = {c0.x, c0.y, c0.z, c0.w};
        const float sn[4] = {s0.x, s0.y, s0.z, s0.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          out[2 * j] = rot(y[2 * j], c[j], -y[2 * j + 1], sn[j]);
          out[2 * j + 1] = rot(y[2 * j + 1], c[j], y[2 * j], sn[j]);
        }
      }
      if (ok[u])
        *reinterpret_cast<uint4*>(p.qkv + t[u] * p.ld + h[u] * D + 8 * g) =
            make_uint4(pack_bf2(out[0], out[1]), pack_bf2(out[2], out[3]), pack_bf2(out[4], out[5]),
                       pack_bf2(out[6], out[7]));
    }
  }
}

template <int D, bool NEOX>
fp8q_status launch_rope(const RopeParams& p, cudaStream_t stream) {
  constexpr int GROUPS = kRopeThreads / (D / 8);
  const int64_t items = p.T * (p.hq + p.hk);
  int64_t blocks = (items + GROUPS * kRopeItems - 1) / (GROUPS * kRopeItems);
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;   // 8 blocks of 256 per SM
  if (blocks > cap) blocks = cap;
  return launch_kernel(qk_norm_rope_kernel<D, NEOX>, dim3(static_cast<unsigned>(blocks)),
                       dim3(kRopeThreads), 0, stream, 1, p);
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_qk_norm_rope(void* qkv, int64_t T, int64_t ld, int num_heads_q,
                                         int num_heads_k, int num_heads_v, int head_dim, float eps,
                                         const void* q_weight, const void* k_weight,
                                         const float* cos_sin_cache, int64_t max_position,
                                         const int64_t* positions, int is_neox, void* stream) {
  if (T < 0 || num_heads_q < 0 || num_heads_k < 0 || num_heads_v < 0) return FP8Q_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return FP8Q_ERR_UNSUPPORTED;
  if (is_neox != 0 && is_neox != 1) return FP8Q_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return FP8Q_ERR_INVALID_ARG;
  const int64_t width = static_cast<int64_t>(num_heads_q + num_heads_k + num_heads_v) * head_dim;
  if (ld < width || ld % 8 != 0 || max_position <= 0) return FP8Q_ERR_INVALID_ARG;
  if (T == 0 || num_heads_q + num_heads_k == 0) return FP8Q_OK;
  if (!qkv || !q_weight || !k_weight || !cos_sin_cache || !positions) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(qkv, 16) || !aligned(q_weight, 16) || !aligned(k_weight, 16) ||
      !aligned(cos_sin_cache, 16) || !aligned(positions, 8))
    return FP8Q_ERR_INVALID_ARG;
  RopeParams p{static_cast<uint16_t*>(qkv), T, ld, num_heads_q, num_heads_k, eps,
               static_cast<const uint16_t*>(q_weight), static_cast<const uint16_t*>(k_weight),
               cos_sin_cache, positions, max_position, device_status_ptr()};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (head_dim * 2 + is_neox) {
    case 128: return launch_rope<64, false>(p, s);
    case 129: return launch_rope<64, true>(p, s);
    case 256: return launch_rope<128, false>(p, s);
    case 257: return launch_rope<128, true>(p, s);
    case 512: return launch_rope<256, false>(p, s);
    default: return launch_rope<256, true>(p, s);
  }
}
