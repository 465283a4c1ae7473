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
#include "fp8q_sm100.cuh"

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
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
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

// Rounding-decision test used by every fast path below.  A fast fp32 value p
// is within a proven relative error e < delta of the exact value v; the two
// ends p(1 - delta) and p(1 + delta) (each one more rounding) bracket v.
// Rounding to nearest is monotone, so if both ends round to the same code, v
// rounds to it as well; otherwise the element takes the exact slow path.
constexpr float kBf16Lo = 1.0f - 0x1p-20f, kBf16Hi = 1.0f + 0x1p-20f;   // errors < 2^-21.7
constexpr float kSiluLo = 1.0f - 0x1p-19f, kSiluHi = 1.0f + 0x1p-19f;   // errors <= 2^-20.6
constexpr float kE4m3Lo = 1.0f - 0x1p-21f, kE4m3Hi = 1.0f + 0x1p-21f;   // errors <= 2^-22
constexpr float kTiny = 0x1p-100f;  // below this fp32 products may lose relative precision

// Two fp32 values -> bf16x2 word (element 0 in the low half), nearest even.
__device__ __forceinline__ uint32_t bf2_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
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

// e^x for |x| <= 87 as 2^(x log2 e) with the exponent split exactly
// (Cody & Waite argument splitting): a = fl(x * L2E) plus the exact FMA
// residual of that product and x times the error of L2E itself; then
// 2^a * (1 + lo ln 2).  Relative error <= 2^-22.2 (measured exhaustively
// over every fp32 x in [-87, 87]).
__device__ __forceinline__ float exp_fast(float x) {
  const float L2E = 1.44269502f;           // fl32(log2 e)
  const float L2E_LO = 1.925963e-8f;       // log2 e - L2E
  const float a = __fmul_rn(x, L2E);
  const float lo = __fmaf_rn(x, L2E_LO, __fmaf_rn(x, L2E, -a));
  const float e = ex2_approx(a);
  return __fmaf_rn(e, __fmul_rn(lo, 0.693147182f), e);
}

// The rare exact paths, kept out of line: inlined into every unrolled element
// position they would overflow the instruction cache.
// r = 1 / sqrt(mean(x^2) + eps) in fp64 from the fp64 row sum of squares.
__device__ __forceinline__ double rms_inv_f64(double ss, int64_t L, float eps) {
  return 1.0 / sqrt(ss / static_cast<double>(L) + static_cast<double>(eps));
}

__device__ __noinline__ uint32_t rms_pair_f64(uint32_t xw, double ss, int64_t L, float eps) {
  const double r = rms_inv_f64(ss, L, eps);
  const uint32_t lo = f64_to_bf16_bits_rn(static_cast<double>(bf16_bits_to_f32(xw & 0xFFFFu)) * r);
  const uint32_t hi = f64_to_bf16_bits_rn(static_cast<double>(bf16_bits_to_f32(xw >> 16)) * r);
  return lo | (hi << 16);
}

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

// RMSNorm pair, fast path: n = bf16(x * r) from p = fl(x * r32) with r32 the
// fp32 rsqrt (relative error < 2^-21.7 in all), bracket +-2^-20.  `unsafe` is set when the
// bracket does not decide the rounding or |p| is tiny; the caller then
// recomputes the pair exactly (rms_pair_f64).
__device__ __forceinline__ uint32_t rms_n_fast(uint32_t xw, float r32, bool& unsafe) {
  const float p0 = __fmul_rn(__uint_as_float(xw << 16), r32);
  const float p1 = __fmul_rn(__uint_as_float(xw & 0xFFFF0000u), r32);
  const uint32_t lo = bf2_rn(__fmul_rn(p0, kBf16Lo), __fmul_rn(p1, kBf16Lo));
  const uint32_t hi = bf2_rn(__fmul_rn(p0, kBf16Hi), __fmul_rn(p1, kBf16Hi));
  unsafe = (lo != hi) || fminf(fabsf(p0), fabsf(p1)) < kTiny;
  return lo;
}

// y = bf16(n * w): one exactly rounded bf16 multiply per half (the product of
// two 8-bit significands is exact before its single rounding).
__device__ __forceinline__ uint32_t bf2_mul(uint32_t n, uint32_t w) {
  const __nv_bfloat162 y = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&n),
                                   *reinterpret_cast<const __nv_bfloat162*>(&w));
  return *reinterpret_cast<const uint32_t*>(&y);
}

// SiLU*mul element, fast: silu(g) * u = g * (1 / (1 + e^-g)) * u with
// exp_fast (<= 2^-22.2), one rounding of 1 + e, rcp_approx (<= 2^-23.3) and
// two multiplications: relative error <= 2^-20.6.
__device__ __forceinline__ float silu_mul_fast(float g, float u) {
  const float d = __fadd_rn(1.0f, exp_fast(-g));
  return __fmul_rn(__fmul_rn(g, rcp_approx(d)), u);
}

// SiLU*mul pair: bracket +-2^-19; gates below -85 (e^-g beyond the fast
// exp's range) and tiny results take the exact path.
__device__ __forceinline__ uint32_t silu_pair_fast(uint32_t gw, uint32_t uw, bool& unsafe) {
  const float g0 = __uint_as_float(gw << 16), g1 = __uint_as_float(gw & 0xFFFF0000u);
  const float p0 = silu_mul_fast(g0, __uint_as_float(uw << 16));
  const float p1 = silu_mul_fast(g1, __uint_as_float(uw & 0xFFFF0000u));
  const uint32_t lo = bf2_rn(__fmul_rn(p0, kSiluLo), __fmul_rn(p1, kSiluLo));
  const uint32_t hi = bf2_rn(__fmul_rn(p0, kSiluHi), __fmul_rn(p1, kSiluHi));
  unsafe = (lo != hi) || fminf(fabsf(p0), fabsf(p1)) < kTiny || fminf(g0, g1) < -85.0f;
  return lo;
}

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

// Codes of a chunk by IEEE division, for the rare chunk whose fast codes
// could differ (out of line).
__device__ __noinline__ uint2 quantize_chunk_ieee(const uint4 y, float s) {
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  uint32_t c[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    c[j] = f2_to_e4m3x2(pk2(__fdiv_rn(bf16_bits_to_f32(w[j] & 0xFFFFu), s),
                            __fdiv_rn(bf16_bits_to_f32(w[j] >> 16), s)));
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// 8 bf16 values (one chunk) -> 8 e4m3 codes of fl32(y / s), fast path:
// t = y * rcp with rcp within 2^-23.3 of 1/s is within 2^-22 of fl32(y/s);
// bracket +-2^-21.  `unsafe` asks the caller for quantize_chunk_ieee.
__device__ __forceinline__ uint2 quantize_chunk_fast(const uint4& y, float rcp, bool& unsafe) {
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  uint32_t c[4];
  bool slow = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float t0 = __fmul_rn(__uint_as_float(w[j] << 16), rcp);
    const float t1 = __fmul_rn(__uint_as_float(w[j] & 0xFFFF0000u), rcp);
    c[j] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(t0, kE4m3Lo), __fmul_rn(t1, kE4m3Lo)), __NV_SATFINITE, __NV_E4M3));
    const uint32_t chi = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(t0, kE4m3Hi), __fmul_rn(t1, kE4m3Hi)), __NV_SATFINITE, __NV_E4M3));
    slow |= c[j] != chi;
  }
  unsafe = slow;
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ float chunk_amax(const uint4& y) {
  // max |y| of 8 bf16 values with packed bf16 max (|.| = sign bits cleared)
  const uint32_t w[4] = {y.x & 0x7FFF7FFFu, y.y & 0x7FFF7FFFu, y.z & 0x7FFF7FFFu, y.w & 0x7FFF7FFFu};
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(w);
  const __nv_bfloat162 m = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
  return fmaxf(__low2float(m), __high2float(m));
}

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Reduction over the T threads of one row team (bar_id 0: the whole CTA with
// __syncthreads; otherwise a named barrier over T threads).  `smem` holds one
// slot per warp; `tid` is the thread's index within the team.
__device__ __forceinline__ void team_sync(int bar_id, int T) {
  if (bar_id == 0) __syncthreads();
  else asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(T) : "memory");
}

template <typename V, typename Op>
__device__ __forceinline__ V team_reduce(V v, Op op, V* smem, int tid, int T, int bar_id) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = tid >> 5, lane = tid & 31, nw = T >> 5;
  team_sync(bar_id, T);  // smem may still be read by a previous reduction
  if (lane == 0) smem[warp] = v;
  team_sync(bar_id, T);
  v = smem[0];
  for (int i = 1; i < nw; ++i) v = op(v, smem[i]);
  return v;
}

struct MaxOp { __device__ float operator()(float a, float b) const { return fmaxf(a, b); } };
struct SumOp { __device__ double operator()(double a, double b) const { return a + b; } };

// Where a row's bf16 input is read from: global memory (streamed, no L1
// allocation) or a shared-memory copy of the row.
struct GlobalRow {
  const uint16_t* base;
  __device__ __forceinline__ uint4 ld(int64_t elem) const { return ld_stream(base + elem); }
};
struct SmemRow {
  const uint16_t* base;
  __device__ __forceinline__ uint4 ld(int64_t elem) const {
    return *reinterpret_cast<const uint4*>(base + elem);
  }
};

// Quantize one row with a team of T threads (T a multiple of 32, CH chunks
// of 8 elements per thread).  `release()` is called once the row's input has
// been read into registers.
template <int OP, bool PER_TOKEN, int CH, typename Src, typename Release>
__device__ __forceinline__ void process_row(const QuantParams& p, int64_t row, const Src& src,
                                            int tid, int T, int bar_id, double* red_d,
                                            float* red_f, Release release) {
  static_assert(CH * 4 <= 32, "one mask bit per bf16 pair");
  const int64_t nchunks = p.L >> 3;
  uint4 y[CH];
  bool valid[CH];
#pragma unroll
  for (int i = 0; i < CH; ++i) valid[i] = (tid + static_cast<int64_t>(i) * T) < nchunks;
  auto off = [&](int i) { return (tid + static_cast<int64_t>(i) * T) * 8; };

  // Hot loops compute every value on the fast path and only flag the rare
  // pairs / chunks whose rounding the fast path cannot decide; the exact
  // recomputation of those runs afterwards, outside the hot loops.
  uint32_t fix = 0;  // bit 4i + j: pair j of chunk i needs the exact path
  if constexpr (OP == OP_PLAIN) {
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (valid[i]) y[i] = src.ld(off(i));
    release();
  } else if constexpr (OP == OP_SILU) {
    // gate and up chunks are read in batches of SB chunks to bound registers.
    constexpr int SB = 2;
#pragma unroll
    for (int i0 = 0; i0 < CH; i0 += SB) {
      uint4 g[SB], u[SB];
#pragma unroll
      for (int i = 0; i < SB; ++i) {
        if (valid[i0 + i]) {
          g[i] = src.ld(off(i0 + i));
          u[i] = src.ld(p.L + off(i0 + i));
        }
      }
#pragma unroll
      for (int i = 0; i < SB; ++i) {
        if (valid[i0 + i]) {
          const uint32_t gw[4] = {g[i].x, g[i].y, g[i].z, g[i].w};
          const uint32_t uw[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            bool bad;
            o[j] = silu_pair_fast(gw[j], uw[j], bad);
            fix |= static_cast<uint32_t>(bad) << (4 * (i0 + i) + j);
          }
          y[i0 + i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    if (fix) {  // rare: re-read the flagged chunks and recompute their pairs exactly
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if ((fix >> (4 * i)) & 0xFu) {
          const uint4 g = src.ld(off(i)), u = src.ld(p.L + off(i));
          uint32_t* yw = reinterpret_cast<uint32_t*>(&y[i]);
          const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
          const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if ((fix >> (4 * i + j)) & 1u) yw[j] = silu_pair_f64(gw[j], uw[j]);
        }
      }
    }
    release();
  } else {  // OP_RMS
    uint4 xv[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (valid[i]) xv[i] = src.ld(off(i));
    release();
    // Sum of squares: squares of bf16 values are exact in fp32; they are
    // accumulated with paired TwoSum (Knuth, TAOCP vol. 2, 4.2.2), a running
    // sum plus the exact error of every addition, then combined in fp64.
    uint64_t sum = pk2(0.0f, 0.0f), comp = pk2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (valid[i]) {
        const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t x2 = bf2_to_f2(xw[j]);
          const uint64_t v = mul2(x2, x2);
          const uint64_t s1 = add2(sum, v);
          const uint64_t bp = sub2(s1, sum);
          comp = add2(comp, add2(sub2(sum, sub2(s1, bp)), sub2(v, bp)));
          sum = s1;
        }
      }
    }
    float s0, s1f, c0, c1;
    up2(sum, s0, s1f);
    up2(comp, c0, c1);
    double ss = (static_cast<double>(s0) + static_cast<double>(s1f)) +
                (static_cast<double>(c0) + static_cast<double>(c1));
    ss = team_reduce(ss, SumOp(), red_d, tid, T, bar_id);
    // Fast path: r32 = rsqrtf(fl32(mean + eps)): <= 2 ulp + half an ulp from
    // the conversion, < 2^-21.9 relative; the fp64 r is computed only by the
    // exact path.
    const float r32 = rsqrtf(static_cast<float>(ss / static_cast<double>(p.L) + static_cast<double>(p.eps)));
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (valid[i]) {
        const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(p.w + off(i)));
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bool bad;
          o[j] = bf2_mul(rms_n_fast(xw[j], r32, bad), ww[j]);
          fix |= static_cast<uint32_t>(bad) << (4 * i + j);
        }
        y[i] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    if (fix) {  // rare: exact bf16(x * r) for the flagged pairs, then y again
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if ((fix >> (4 * i)) & 0xFu) {
          const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
          const uint4 wv = __ldg(reinterpret_cast<const uint4*>(p.w + off(i)));
          const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
          uint32_t* yw = reinterpret_cast<uint32_t*>(&y[i]);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if ((fix >> (4 * i + j)) & 1u) yw[j] = bf2_mul(rms_pair_f64(xw[j], ss, p.L, p.eps), ww[j]);
        }
      }
    }
  }

  // Codes are stored as soon as they are made; a flagged chunk is stored
  // again, from IEEE division, after the loop.
  uint8_t* qr = p.q + row * p.ldq;
  uint32_t qfix = 0;  // bit i: chunk i needs IEEE division
  if constexpr (PER_TOKEN) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (valid[i]) amax = fmaxf(amax, chunk_amax(y[i]));
    amax = team_reduce(amax, MaxOp(), red_f, tid, T, bar_id);
    const float s = group_scale(amax, p.ue8m0);
    const float rcp = rcp_approx(s);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (valid[i]) {
        bool bad;
        *reinterpret_cast<uint2*>(qr + off(i)) = quantize_chunk_fast(y[i], rcp, bad);
        qfix |= static_cast<uint32_t>(bad) << i;
      }
    }
    if (tid == 0) p.s[row * p.s_sm] = s;
    if (qfix) {
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if ((qfix >> i) & 1u) *reinterpret_cast<uint2*>(qr + off(i)) = quantize_chunk_ieee(y[i], s);
    }
  } else {
    // 128-wide groups: the 16 threads tid & ~15 .. +15 own one group per i
    // (T is a multiple of 32 and L of 128, so whole half-warps are valid or not).
    float sc[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      float a = valid[i] ? chunk_amax(y[i]) : 0.0f;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      sc[i] = group_scale(a, p.ue8m0);
      if (valid[i]) {
        bool bad;
        *reinterpret_cast<uint2*>(qr + off(i)) = quantize_chunk_fast(y[i], rcp_approx(sc[i]), bad);
        qfix |= static_cast<uint32_t>(bad) << i;
        if ((tid & 15) == 0) p.s[row * p.s_sm + (off(i) >> 7) * p.s_sg] = sc[i];
      }
    }
    if (qfix) {
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if ((qfix >> i) & 1u) *reinterpret_cast<uint2*>(qr + off(i)) = quantize_chunk_ieee(y[i], sc[i]);
    }
  }
}

// Register kernel: one CTA per row, the row loaded straight into registers.
// Used for rows too long for the shared-memory ring below.
template <int OP, bool PER_TOKEN, int CH>
__global__ void __launch_bounds__(kMaxThreads, (CH <= 4 ? 2 : 1)) quant_rows_kernel(const QuantParams p) {
  __shared__ double red_d[32];
  __shared__ float red_f[32];
  for (int64_t row = blockIdx.x; row < p.M; row += gridDim.x)
    process_row<OP, PER_TOKEN, CH>(p, row, GlobalRow{p.x + row * p.ldx}, threadIdx.x, blockDim.x,
                                   0, red_d, red_f, [] {});
}

// Ring kernel: persistent CTAs; warp 0 (one lane) streams whole input rows
// into a ring of NBUF shared-memory buffers with cp.async.bulk (completion on
// the slot's mbarrier), while NT teams of T compute threads each quantize a
// different row from shared memory (team t takes the CTA's rows i = t, t+NT,
// ...; NBUF is a multiple of NT, so a slot always serves the same team).  HBM
// reads stay in flight independently of the compute.  Every wait is bounded; a
// wait that gives up records FP8Q_ERR_TIMEOUT, the team leaves together (vote
// on its named barrier) and the producer lets its copies land.
constexpr int kRingMaxBuf = 16;

// CTA size cap of the ring kernel (it sets the register budget per thread):
// SiLU needs more registers than the other ops, 8 chunks per thread more still.
__host__ __device__ constexpr int ring_max_threads(int op, int ch) {
  return ch == 8 ? 512 : (op == OP_SILU ? 800 : 1024);
}

template <int OP, bool PER_TOKEN, int CH>
__global__ void __launch_bounds__(ring_max_threads(OP, CH), 1)
    quant_ring_kernel(const QuantParams p, int nbuf, int nteams, int T, int row_stride_bytes,
                      int* status) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kRingMaxBuf], empty[kRingMaxBuf];
  __shared__ double red_d[8][32];
  __shared__ float red_f[8][32];
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t copy_bytes = static_cast<uint32_t>((OP == OP_SILU ? 4 : 2) * p.L);

  if (threadIdx.x == 0) {
    for (int i = 0; i < nbuf; ++i) {
      sm100::mbar_init(&full[i], 1);
      sm100::mbar_init(&empty[i], T / 32);
    }
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      for (int64_t row = blockIdx.x; row < p.M; row += gridDim.x, ++i) {
        const int slot = i % nbuf;
        if (!sm100::mbar_wait(&empty[slot], ((i / nbuf) & 1) ^ 1u, &abort_flag, status)) {
          ok = false;
          break;
        }
        sm100::mbar_arrive_expect_tx(&full[slot], copy_bytes);
        sm100::bulk_load(ring + static_cast<size_t>(slot) * row_stride_bytes, p.x + row * p.ldx,
                         copy_bytes, &full[slot]);
      }
      if (!ok) {
        const int first = i - nbuf > 0 ? i - nbuf : 0;
        for (int j = first; j < i; ++j) sm100::drain_wait(&full[j % nbuf], (j / nbuf) & 1);
      }
    }
    return;
  }

  const int team = (threadIdx.x - 32) / T;
  const int tid = (threadIdx.x - 32) - team * T;
  const int bar = 1 + team;
  int i = team;
  for (int64_t row = blockIdx.x + static_cast<int64_t>(team) * gridDim.x; row < p.M;
       row += static_cast<int64_t>(nteams) * gridDim.x, i += nteams) {
    const int slot = i % nbuf;
    const bool ok = sm100::mbar_wait(&full[slot], (i / nbuf) & 1, &abort_flag, status);
    if (sm100::team_any(!ok, bar, T)) break;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(ring + static_cast<size_t>(slot) * row_stride_bytes);
    process_row<OP, PER_TOKEN, CH>(p, row, SmemRow{src}, tid, T, bar, red_d[team], red_f[team], [&] {
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&empty[slot]);
    });
  }
}

// Threads per row: enough that CH chunks per thread cover the row; a multiple
// of 32 (whole warps), at least 32.
inline int threads_for(int64_t nchunks, int ch) {
  int64_t t = (nchunks + ch - 1) / ch;
  t = ((t + 31) / 32) * 32;
  return static_cast<int>(t < 32 ? 32 : t);
}

constexpr int kRingSmemMax = 200 * 1024;   // ring bytes per CTA (one CTA per SM)

// Ring geometry: as many teams as fit the CTA size cap (at most 8), and
// the deepest ring (a multiple of the team count, >= 2 slots per team) that
// fits the shared memory.  Returns false when even one team with two slots
// does not fit.
bool ring_geometry(int64_t row_bytes, int T, int max_threads, int* nteams, int* nbuf, int* stride) {
  *stride = static_cast<int>(((row_bytes + 127) / 128) * 128);
  int nt = (max_threads - 32) / T;
  nt = nt > 8 ? 8 : nt;
  while (nt >= 1 && 2LL * nt * *stride > kRingSmemMax) --nt;
  if (nt < 1) return false;
  int per = static_cast<int>(kRingSmemMax / (static_cast<int64_t>(nt) * *stride));
  if (per * nt > kRingMaxBuf) per = kRingMaxBuf / nt;
  if (per < 2) return false;
  *nteams = nt;
  *nbuf = per * nt;
  return true;
}

template <int OP, bool PER_TOKEN, int CH>
fp8q_status launch_ring(const QuantParams& p, int T, int nteams, int nbuf, int stride,
                        cudaStream_t stream) {
  const int smem = nbuf * stride;
  auto kern = quant_ring_kernel<OP, PER_TOKEN, CH>;
  static int attr_done[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr_done[dev] = 1;
  }
  int64_t grid = num_sms();
  if (grid > p.M) grid = p.M;
  kern<<<static_cast<unsigned>(grid), 32 + nteams * T, smem, stream>>>(p, nbuf, nteams, T, stride,
                                                                       device_status_ptr());
  return launch_status();
}

template <int OP>
fp8q_status launch_quant(const QuantParams& p, cudaStream_t stream) {
  if (p.M == 0) return FP8Q_OK;
  const int64_t nchunks = p.L / 8;
  const bool per_token = p.group == p.L;
  // 4 chunks (32 elements) per thread while that needs <= 512 threads, else 8.
  const int ch = nchunks > 4 * kMaxThreads ? 8 : 4;
  const int T = threads_for(nchunks, ch);
  if (T > kMaxThreads) return FP8Q_ERR_UNSUPPORTED;
  // Long rows (8 chunks per thread) stream through the shared-memory ring;
  // shorter rows run many CTAs per SM on registers alone.
  const int64_t row_bytes = (OP == OP_SILU ? 4 : 2) * p.L;
  int nteams = 0, nbuf = 0, stride = 0;
  // (Measured: for rows of <= 2048 chunks the register kernel, with many
  // CTAs per SM, is faster than the ring.)
  if (ch == 8 && ring_geometry(row_bytes, T, ring_max_threads(OP, ch), &nteams, &nbuf, &stride))
    return per_token ? launch_ring<OP, true, 8>(p, T, nteams, nbuf, stride, stream)
                     : launch_ring<OP, false, 8>(p, T, nteams, nbuf, stride, stream);
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
