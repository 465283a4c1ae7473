// fp8q_quant_math.cuh -- the arithmetic of dynamic FP8 / int8 activation
// quantization shared by the quant kernels and the GEMM epilogue that fuses
// SiLU*mul quant: packed fp32 pair helpers, the exact group scale and codes
// (Markstein's division step), the exact RMSNorm and SiLU*mul brackets with
// their fp64 cold paths.  See fp8q_quant.cu for the definitions they meet.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp8q_common.cuh"

namespace fp8q {
namespace {   // internal linkage in every translation unit that includes it

// ---------------------------------------------------------------------------
// Scalar helpers

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

// Hardware approximations with error bounds measured exhaustively (every
// fp32 input of the ranges used, against fp64): ex2.approx.ftz <= 2^-22.7
// relative on [-126, 128); rcp.approx.ftz <= 2^-23.3 relative.
__device__ __forceinline__ float ex2_approx(float a) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}
__device__ __forceinline__ float rcp_approx(float s) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
  return r;
}

// ---------------------------------------------------------------------------
// Paired fp32 arithmetic (sm_100 .f32x2: two IEEE fp32 operations per
// instruction).  A pair travels as one 64-bit register: low word = element 0.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t dup2(float v) { return pk2(v, v); }
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mulz2(uint64_t a, uint64_t b) {   // toward zero
  uint64_t r;
  asm("mul.rz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// Both elements one unit in the last place further from zero (finite
// values: the bit patterns are sign-magnitude, and no carry crosses lanes).
__device__ __forceinline__ uint64_t bump2(uint64_t v) { return v + 0x0000000100000001ull; }

// bf16x2 word (element 0 in the low half) <-> fp32 pair.
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
  return pk2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2_rn(uint64_t v) {
  float a, b;
  up2(v, a, b);
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t f2_to_e4m3x2(uint64_t v) {
  float a, b;
  up2(v, a, b);
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// y = bf16(n * w): one exactly rounded bf16 multiply per half (the product of
// two 8-bit significands is exact before its single rounding).
__device__ __forceinline__ uint32_t bf2_mul(uint32_t n, uint32_t w) {
  const __nv_bfloat162 y = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&n),
                                   *reinterpret_cast<const __nv_bfloat162*>(&w));
  return *reinterpret_cast<const uint32_t*>(&y);
}

// max |y| of 8 bf16 values, accumulated packed (|.| = sign bits cleared).
__device__ __forceinline__ uint32_t chunk_absmax2(const uint4& y, uint32_t m) {
  const uint32_t w[4] = {y.x & 0x7FFF7FFFu, y.y & 0x7FFF7FFFu, y.z & 0x7FFF7FFFu, y.w & 0x7FFF7FFFu};
  __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&m);
#pragma unroll
  for (int k = 0; k < 4; ++k) a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162*>(&w[k]));
  return *reinterpret_cast<const uint32_t*>(&a);
}
__device__ __forceinline__ float absmax2_to_f32(uint32_t m) {
  return fmaxf(bf16_bits_to_f32(m & 0xFFFFu), bf16_bits_to_f32(m >> 16));
}

// ---------------------------------------------------------------------------
// Scales and codes

// Scale of a group: fl32(max(amax, 1e-10) / 448), UE8M0: rounded up to a
// power of two.  The quotient is q0 = a * fl(1/448) corrected once by its
// exact FMA residual (Markstein's correction step); amax is a bf16 value, and
// the GPU tests check this against IEEE division for every positive bf16 amax.
constexpr float kInv448 = 1.0f / 448.0f;

__device__ __forceinline__ float group_scale(float amax, int ue8m0) {
  const float a = fmaxf(amax, 1e-10f);
  const float q0 = __fmul_rn(a, kInv448);
  const float r = __fmaf_rn(-448.0f, q0, a);
  float s = __fmaf_rn(r, kInv448, q0);
  if (ue8m0) {
    uint32_t u = __float_as_uint(s);          // s >= 2.2e-13: a positive normal
    if (u & 0x007FFFFFu) u = (u & 0xFF800000u) + 0x00800000u;
    s = __uint_as_float(u);
  }
  return s;
}

// A scale with what the codes need: the correctly rounded reciprocal
// rcp = RN(1/s) and -s, both duplicated into pairs.
struct QScale {
  float s;
  uint64_t rcp2, neg2;
};
__device__ __forceinline__ QScale make_qscale(float amax, int ue8m0, int i8 = 0) {
  QScale q;
  // int8 codes: s = fl32(max(amax, 1e-10) / 127), IEEE division
  q.s = i8 ? __fdiv_rn(fmaxf(amax, 1e-10f), 127.0f) : group_scale(amax, ue8m0);
  q.rcp2 = dup2(__frcp_rn(q.s));
  q.neg2 = dup2(-q.s);
  return q;
}

// 8 bf16 values (one chunk) -> 8 e4m3 codes of fl32(y / s).  The quotient is
// the IEEE one, by Markstein's division step (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990): q0 = RN(y rcp) is within an ulp of y/s, so the residual
// r = y - q0 s is exact under FMA and RN(q0 + r rcp) = RN(y/s) when rcp is
// the correctly rounded 1/s.  (Quotients too small for that argument, below
// 2^-12, become code 0 either way.)  Ties of the e4m3 rounding -- frequent:
// bf16 data over a bf16 amax often gives quotients like 10.5 exactly -- are
// then decided by the conversion itself, as in the definition.
__device__ __forceinline__ uint2 quant_chunk(const uint4& y, const QScale& qs) {
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint64_t f = bf2_to_f2(w[k]);
    const uint64_t q0 = mul2(f, qs.rcp2);
    const uint64_t r = fma2(q0, qs.neg2, f);
    c[k] = f2_to_e4m3x2(fma2(r, qs.rcp2, q0));
  }
  // The step turns y = -0 into +0; every code takes the sign bit of its y
  // (bytes 1 and 3 of each bf16x2 word hold the two signs in their bit 7).
  return make_uint2((c[0] | (c[1] << 16)) | (__byte_perm(w[0], w[1], 0x7531) & 0x80808080u),
                    (c[2] | (c[3] << 16)) | (__byte_perm(w[2], w[3], 0x7531) & 0x80808080u));
}

// 8 bf16 values -> 8 int8 codes: the same IEEE quotient fl32(y / s) as
// quant_chunk, rounded to the nearest integer, ties to even (cvt.rni; |y/s|
// <= 127 by the choice of s, NaN gives 0).
__device__ __forceinline__ int32_t f32_to_i32_rni(float v) {
  int32_t r;
  asm("cvt.rni.s32.f32 %0, %1;" : "=r"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint2 quant_chunk_i8(const uint4& y, const QScale& qs) {
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  uint32_t c[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint64_t f = bf2_to_f2(w[k]);
    const uint64_t q0 = mul2(f, qs.rcp2);
    const uint64_t r = fma2(q0, qs.neg2, f);
    float a, b;
    up2(fma2(r, qs.rcp2, q0), a, b);
    c[k] = __byte_perm(static_cast<uint32_t>(f32_to_i32_rni(a)), static_cast<uint32_t>(f32_to_i32_rni(b)),
                       0x0040);                          // low bytes of both -> bytes 0, 1
  }
  return make_uint2(__byte_perm(c[0], c[1], 0x5410), __byte_perm(c[2], c[3], 0x5410));
}

// ---------------------------------------------------------------------------
// RMSNorm

// r = 1 / sqrt(mean(x^2) + eps) in fp64 from the fp64 row sum of squares.
__device__ __forceinline__ double rms_inv_f64(double ss, int64_t L, float eps) {
  return 1.0 / sqrt(ss / static_cast<double>(L) + static_cast<double>(eps));
}

// Exact bf16(x * r) of a pair (out of line).
__device__ __noinline__ uint32_t rms_pair_f64(uint32_t xw, double ss, int64_t L, float eps) {
  const double r = rms_inv_f64(ss, L, eps);
  const uint32_t lo = f64_to_bf16_bits_rn(static_cast<double>(bf16_bits_to_f32(xw & 0xFFFFu)) * r);
  const uint32_t hi = f64_to_bf16_bits_rn(static_cast<double>(bf16_bits_to_f32(xw >> 16)) * r);
  return lo | (hi << 16);
}

// n = bf16(x * r) of a pair, from the bracket ends a = rz(x r_lo) and
// b = rz(x r_hi) + 1 ulp (r_lo <= r <= r_hi): |a| <= |x r| <= |b|.  Returns the
// rounding of a; `d` collects the XOR with the rounding of b.
__device__ __forceinline__ uint32_t rms_n_pair(uint32_t xw, uint64_t rlo2, uint64_t rhi2, uint32_t& d) {
  const uint64_t f = bf2_to_f2(xw);
  const uint32_t na = f2_to_bf2_rn(mulz2(f, rlo2));
  d |= na ^ f2_to_bf2_rn(bump2(mulz2(f, rhi2)));
  return na;
}

// Cold path of a flagged RMSNorm chunk: the pairs whose bracket is open get
// the exact bf16(x r), then y = bf16(n w).
__device__ __noinline__ uint4 rms_chunk_fix(const uint4 xv, const uint4 wv, uint4 y, uint64_t rlo2,
                                           uint64_t rhi2, double ss, int64_t L, float eps) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
  uint32_t yw[4] = {y.x, y.y, y.z, y.w};
  for (int k = 0; k < 4; ++k) {
    uint32_t d = 0;
    rms_n_pair(xw[k], rlo2, rhi2, d);
    if (d) yw[k] = bf2_mul(rms_pair_f64(xw[k], ss, L, eps), ww[k]);
  }
  return make_uint4(yw[0], yw[1], yw[2], yw[3]);
}

// r = 1/sqrt(m) in fp64: rsqrtf, one Newton step in fp64 (error
// <= 1.5 e^2 + fp64 roundings, e <= 2^-21 the rsqrtf error: below 2^-40).
__device__ __forceinline__ double rms_r1(double m) {
  if (m >= 0x1p-120 && m <= 0x1p120) {
    const double r0 = static_cast<double>(rsqrtf(static_cast<float>(m)));
    const double h = __fma_rn(-m * r0, r0, 1.0);          // 1 - m r0^2
    return __fma_rn(0.5 * r0, h, r0);
  }
  return 1.0 / sqrt(m);
}

// fp32 bracket of r = r1 (1 +- rel): the fp32 values just below and above.
__device__ __forceinline__ void rms_bracket_of(double r1, double rel, float& r_lo, float& r_hi) {
  r_lo = __double2float_rd(r1 * (1.0 - rel));
  r_hi = __double2float_ru(r1 * (1.0 + rel));
}

// Fast bracket of r = 1/sqrt(m) for an exact m: 1 -+ 2^-30 around rms_r1.
__device__ __forceinline__ void rms_bracket(double m, float& r_lo, float& r_hi) {
  rms_bracket_of(rms_r1(m), 0x1p-30, r_lo, r_hi);
}

// ---------------------------------------------------------------------------
// SiLU * mul

// Bracket of the fast SiLU*mul value p (relative error <= 2^-21.0, below):
// p (1 -+ 2^-20.5), each end one more rounding.
constexpr float kSiluLo = 1.0f - 0x1.6a09e6p-21f, kSiluHi = 1.0f + 0x1.6a09e6p-21f;
constexpr float kTiny = 0x1p-100f;  // below this fp32 products may lose relative precision

// e^-g for a pair, |g| <= 85: 2^(-g log2 e) with the exponent split exactly
// (Cody & Waite argument splitting): a = fl(g L2E) plus the exact FMA
// residual of that product and g times the error of L2E itself; then
// 2^-a (1 + lo ln 2).  Relative error <= 2^-22.2 (measured exhaustively for
// every fp32 argument in [-87, 87] by the tests).
__device__ __forceinline__ uint64_t exp_neg2(uint64_t g2) {
  const float L2E = 1.44269502f;           // fl32(log2 e)
  const float L2E_LO = 1.925963e-8f;       // log2 e - L2E
  const uint64_t am = mul2(g2, dup2(L2E));                   // fl(g L2E)
  const uint64_t r = fma2(g2, dup2(-L2E), am);               // -(g L2E - am), exact
  const uint64_t lo = fma2(g2, dup2(-L2E_LO), r);
  float a0, a1;
  up2(am, a0, a1);
  const uint64_t e = pk2(ex2_approx(-a0), ex2_approx(-a1));
  return fma2(e, mul2(lo, dup2(0.693147182f)), e);
}

// Fast silu(g) * u of a pair: g * (1 / (1 + e^-g)) * u with exp_neg2
// (<= 2^-22.2), one rounding of 1 + e, the Newton-refined reciprocal
// (<= 2^-23.9) and two multiplications: relative error <= 2^-21.0 while
// nothing is tiny and the gate is >= -85 (within the fast exp's range).
__device__ __forceinline__ uint64_t silu_p2(uint64_t g2, uint64_t u2) {
  const uint64_t dd = add2(dup2(1.0f), exp_neg2(g2));
  float d0, d1;
  up2(dd, d0, d1);
  // -1/d by rcp.approx of -d, then one Newton step: h = 1 - d r0,
  // -r1 = -r0 (1 + h); the result is within 2^-23.9 of 1/d.
  const uint64_t nr0 = pk2(rcp_approx(-d0), rcp_approx(-d1));
  const uint64_t h = fma2(dd, nr0, dup2(1.0f));
  const uint64_t nr1 = fma2(nr0, h, nr0);
  // (-g)(-r1) u: negate g by its sign bits
  return mul2(mul2(g2 ^ 0x8000000080000000ull, nr1), u2);
}

// bf16 rounding of the low bracket end of a pair; `d` collects its XOR with
// the high end; `bad` is set for tiny values, tiny gates (g (1/(1+e^-g)) would
// be an fp32 subnormal short of bits, which a large up value can lift back into
// range) and gates below -85.
__device__ __forceinline__ uint32_t silu_pair(uint32_t gw, uint32_t uw, uint32_t& d, bool& bad) {
  const uint64_t g2 = bf2_to_f2(gw);
  const uint64_t p = silu_p2(g2, bf2_to_f2(uw));
  const uint32_t na = f2_to_bf2_rn(mul2(p, dup2(kSiluLo)));
  d |= na ^ f2_to_bf2_rn(mul2(p, dup2(kSiluHi)));
  float p0, p1, g0, g1;
  up2(p, p0, p1);
  up2(g2, g0, g1);
  bad |= fminf(fminf(fabsf(p0), fabsf(p1)), fminf(fabsf(g0), fabsf(g1))) < kTiny || fminf(g0, g1) < -85.0f;
  return na;
}

// Exact bf16(silu(g) * u) of a pair (out of line).
__device__ __noinline__ uint32_t silu_pair_f64(uint32_t gw, uint32_t uw) {
  uint32_t out = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const double g = bf16_bits_to_f32((gw >> (16 * h)) & 0xFFFFu);
    const double u = bf16_bits_to_f32((uw >> (16 * h)) & 0xFFFFu);
    out |= f64_to_bf16_bits_rn(g / (1.0 + exp(-g)) * u) << (16 * h);
  }
  return out;
}

// Cold path of a flagged SiLU chunk: each element whose fast value is not
// proven is recomputed exactly.  A zero gate or up value makes the fast
// value an exact (signed) zero, so those results are kept.
__device__ __noinline__ uint4 silu_chunk_fix(const uint4 g, const uint4 u, uint4 y) {
  const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
  uint32_t yw[4] = {y.x, y.y, y.z, y.w};
  for (int k = 0; k < 4; ++k) {
    const uint64_t g2 = bf2_to_f2(gw[k]), u2 = bf2_to_f2(uw[k]);
    const uint64_t p = silu_p2(g2, u2);
    const uint32_t open = f2_to_bf2_rn(mul2(p, dup2(kSiluLo))) ^ f2_to_bf2_rn(mul2(p, dup2(kSiluHi)));
    float pf[2], gf[2], uf[2];
    up2(p, pf[0], pf[1]);
    up2(g2, gf[0], gf[1]);
    up2(u2, uf[0], uf[1]);
    bool need = open != 0;
    for (int h = 0; h < 2; ++h)
      need |= gf[h] < -85.0f ||
              ((fabsf(pf[h]) < kTiny || fabsf(gf[h]) < kTiny) && gf[h] != 0.0f && uf[h] != 0.0f);
    if (need) yw[k] = silu_pair_f64(gw[k], uw[k]);
  }
  return make_uint4(yw[0], yw[1], yw[2], yw[3]);
}

// ---------------------------------------------------------------------------
// Fast y (SiLU*mul per token, the default mode).  y comes within one bf16
// step of its definition (differing only when the real value lies closer to a
// bf16 rounding midpoint than the fast value's error); the quant kernels
// recompute exactly the elements that can decide a group's amax, so scales
// stay exact and codes (from the exact IEEE quotient of y) differ only where
// y does.

// Fast bf16(silu(g) u) of a pair: (g u) / (1 + 2^(-g log2 e)) with ex2.approx
// and rcp.approx.  For gates >= -85: the product g u is exact unless it
// under- or overflows; the rounding of the exponent argument costs a relative
// error of at most |g| 2^-23.5 ln 2 in 2^(.) (<= 2^-17.3), ex2.approx
// 2^-22.7, 1 + e one rounding, rcp.approx 2^-23.3, the last product one
// rounding: |error| <= 2^-17 relative, far below a bf16 step (2^-8); a tiny
// or overflowing g u gives a value within a step of the rounded real one or
// the flagged infinity.  Gates below -85 (2^(.) overflowing) are the caller's
// to send to the exact path.
__device__ __forceinline__ uint32_t silu_pair_fast(uint32_t gw, uint32_t uw) {
  const float NL2E = -1.44269502f;          // -fl32(log2 e)
  const uint64_t g2 = bf2_to_f2(gw);
  float a0, a1;
  up2(mul2(g2, dup2(NL2E)), a0, a1);
  float d0, d1;
  up2(add2(dup2(1.0f), pk2(ex2_approx(a0), ex2_approx(a1))), d0, d1);
  return f2_to_bf2_rn(mul2(mul2(g2, bf2_to_f2(uw)), pk2(rcp_approx(d0), rcp_approx(d1))));
}

// Lowest gate of a chunk (packed bf16 minimum of its eight gate values; a NaN
// gate is ignored, as the exact path's < -85 test ignores it).
__device__ __forceinline__ float chunk_min_gate(const uint4& g) {
  __nv_bfloat162 m = *reinterpret_cast<const __nv_bfloat162*>(&g.x);
  m = __hmin2(m, *reinterpret_cast<const __nv_bfloat162*>(&g.y));
  m = __hmin2(m, *reinterpret_cast<const __nv_bfloat162*>(&g.z));
  m = __hmin2(m, *reinterpret_cast<const __nv_bfloat162*>(&g.w));
  return fminf(__low2float(m), __high2float(m));
}

// Candidate margin of the fast SiLU*mul: a fast y lies within one bf16 step
// of its definition, so the exact amax of a group is the exact value of an
// element whose fast value is within one step of the fast amax, and no element
// more than 4 steps below it can reach that (a margin of two steps to spare).
constexpr uint32_t kCandSteps = 4;

// The bf16 magnitude `steps` below a (a bf16 value as fp32, >= 0; 0 stays 0):
// consecutive bf16 magnitudes are consecutive integers.
__device__ __forceinline__ float bf16_steps_below(float a, uint32_t steps) {
  const uint32_t b = __float_as_uint(a) >> 16;
  return __uint_as_float((b > steps ? b - steps : 0u) << 16);
}

}  // namespace
}  // namespace fp8q
