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
constexpr float kBf16Lo = 1.0f - 0x1p-20f, kBf16Hi = 1.0f + 0x1p-20f;   // errors <= 2^-21
constexpr float kE4m3Lo = 1.0f - 0x1p-21f, kE4m3Hi = 1.0f + 0x1p-21f;   // errors <= 2^-22

// Either bf16 half nonzero with |v| < 2^-100: fp32 products there may have
// lost relative precision, so the bracket is not trusted.
__device__ __forceinline__ bool bf2_tiny(uint32_t h) {
  const uint32_t e = h & 0x7F807F80u;
  return __vcmpltu2(__vsub2(e, 0x00800080u), 0x0D000D00u) != 0u;
}

// The rare exact paths, kept out of line: inlined into every unrolled element
// position they would overflow the instruction cache.
__device__ __noinline__ uint32_t rms_pair_f64(uint32_t xw, double r) {
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

// RMSNorm pair: n = bf16(x * r), y = bf16(n * w).  Fast path: p = fl(x * fl(r)),
// relative error <= 2^-23 (two roundings); bracket +-2^-20.  n * w is one
// exactly rounded bf16 multiply (the product of two 8-bit significands is
// exact before its single rounding).
__device__ __forceinline__ uint32_t rms_pair(uint32_t xw, uint32_t ww, uint64_t r2, double r) {
  const uint64_t p = mul2(bf2_to_f2(xw), r2);
  const uint32_t nlo = f2_to_bf2_rn(mul2(p, pk2(kBf16Lo, kBf16Lo)));
  const uint32_t nhi = f2_to_bf2_rn(mul2(p, pk2(kBf16Hi, kBf16Hi)));
  const uint32_t n = (nlo == nhi && !bf2_tiny(nlo)) ? nlo : rms_pair_f64(xw, r);
  const __nv_bfloat162 y = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&n),
                                   *reinterpret_cast<const __nv_bfloat162*>(&ww));
  return *reinterpret_cast<const uint32_t*>(&y);
}

// SiLU*mul pair: y = bf16(silu(g) * u), silu(g) = g / (1 + e^-g) evaluated
// as g * fl(1/fl(1 + e)) * u.  Error of the fp32 value: expf <= 2 ulp
// (2^-22 relative), then four IEEE roundings: <= 2^-21; bracket +-2^-20.
// Gates below -85 make e^-g overflow fp32: always the exact path.
__device__ __forceinline__ uint32_t silu_pair(uint32_t gw, uint32_t uw) {
  const float g0 = __uint_as_float(gw << 16), g1 = __uint_as_float(gw & 0xFFFF0000u);
  const uint64_t d = add2(pk2(expf(-g0), expf(-g1)), pk2(1.0f, 1.0f));
  float d0, d1;
  up2(d, d0, d1);
  const uint64_t sl = mul2(pk2(g0, g1), pk2(__frcp_rn(d0), __frcp_rn(d1)));
  const uint64_t p = mul2(sl, bf2_to_f2(uw));
  const uint32_t lo = f2_to_bf2_rn(mul2(p, pk2(kBf16Lo, kBf16Lo)));
  const uint32_t hi = f2_to_bf2_rn(mul2(p, pk2(kBf16Hi, kBf16Hi)));
  if (lo != hi || bf2_tiny(lo) || fminf(g0, g1) < -85.0f) return silu_pair_f64(gw, uw);
  return lo;
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

// 8 bf16 values (one chunk) -> 8 e4m3 codes of fl32(y / s).  Fast path:
// t = y * fl(1/s) is within 1.5 * 2^-23 of fl32(y/s); bracket +-2^-21.
// `rcp` = __frcp_rn(s).
__device__ __forceinline__ uint2 quantize_chunk(const uint4& y, float s, float rcp) {
  const uint32_t w[4] = {y.x, y.y, y.z, y.w};
  const uint64_t r2 = pk2(rcp, rcp);
  uint32_t c[4];
  bool slow = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint64_t t = mul2(bf2_to_f2(w[j]), r2);
    c[j] = f2_to_e4m3x2(mul2(t, pk2(kE4m3Lo, kE4m3Lo)));
    slow |= c[j] != f2_to_e4m3x2(mul2(t, pk2(kE4m3Hi, kE4m3Hi)));
  }
  if (slow) return quantize_chunk_ieee(y, s);
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__device__ __forceinline__ float chunk_amax(const uint4& y) {
  // |bf16| max on the bit patterns (sign cleared; magnitudes order as
  // integers), two halves per SIMD max.
  uint32_t m = __vmaxu2(y.x & 0x7FFF7FFFu, y.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, __vmaxu2(y.z & 0x7FFF7FFFu, y.w & 0x7FFF7FFFu));
  return bf16_bits_to_f32(max(m & 0xFFFFu, m >> 16));
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
  const int64_t nchunks = p.L >> 3;
  uint4 y[CH];
  bool valid[CH];
#pragma unroll
  for (int i = 0; i < CH; ++i) valid[i] = (tid + static_cast<int64_t>(i) * T) < nchunks;

  if constexpr (OP == OP_PLAIN) {
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (valid[i]) y[i] = src.ld((tid + static_cast<int64_t>(i) * T) * 8);
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
          const int64_t off = (tid + static_cast<int64_t>(i0 + i) * T) * 8;
          g[i] = src.ld(off);
          u[i] = src.ld(p.L + off);
        }
      }
#pragma unroll
      for (int i = 0; i < SB; ++i) {
        if (valid[i0 + i]) {
          const uint32_t gw[4] = {g[i].x, g[i].y, g[i].z, g[i].w};
          const uint32_t uw[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
          uint32_t o[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) o[j] = silu_pair(gw[j], uw[j]);
          y[i0 + i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
    release();
  } else {  // OP_RMS
    uint4 xv[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (valid[i]) xv[i] = src.ld((tid + static_cast<int64_t>(i) * T) * 8);
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
    const double r = 1.0 / sqrt(ss / static_cast<double>(p.L) + static_cast<double>(p.eps));
    const uint64_t r2 = pk2(static_cast<float>(r), static_cast<float>(r));
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (valid[i]) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(p.w + (tid + static_cast<int64_t>(i) * T) * 8));
        const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = rms_pair(xw[j], ww[j], r2, r);
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
    amax = team_reduce(amax, MaxOp(), red_f, tid, T, bar_id);
    const float s = group_scale(amax, p.ue8m0);
    const float rcp = __frcp_rn(s);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (valid[i]) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        *reinterpret_cast<uint2*>(qr + c * 8) = quantize_chunk(y[i], s, rcp);
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
        *reinterpret_cast<uint2*>(qr + c * 8) = quantize_chunk(y[i], s, __frcp_rn(s));
        if ((tid & 15) == 0) p.s[row * p.s_sm + (c >> 4) * p.s_sg] = s;
      }
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
// the slot's mbarrier), so HBM reads stay in flight while the T compute
// threads quantize earlier rows from shared memory.  Every wait is bounded; a
// wait that gives up records FP8Q_ERR_TIMEOUT, the compute team leaves
// together (vote on a named barrier) and the producer lets its copies land.
constexpr int kRingMaxBuf = 8;

template <int OP, bool PER_TOKEN, int CH>
__global__ void __launch_bounds__(kMaxThreads + 32, 1)
    quant_ring_kernel(const QuantParams p, int nbuf, int row_stride_bytes, int* status) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kRingMaxBuf], empty[kRingMaxBuf];
  __shared__ double red_d[32];
  __shared__ float red_f[32];
  __shared__ volatile int abort_flag;
  const int T = blockDim.x - 32;
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

  const int tid = threadIdx.x - 32;
  int i = 0;
  for (int64_t row = blockIdx.x; row < p.M; row += gridDim.x, ++i) {
    const int slot = i % nbuf;
    const bool ok = sm100::mbar_wait(&full[slot], (i / nbuf) & 1, &abort_flag, status);
    if (sm100::team_any(!ok, 1, T)) break;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(ring + static_cast<size_t>(slot) * row_stride_bytes);
    process_row<OP, PER_TOKEN, CH>(p, row, SmemRow{src}, tid, T, 1, red_d, red_f, [&] {
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

constexpr int kRingSmemTarget = 96 * 1024;    // ring bytes aimed at per CTA
constexpr int kRingSmemMax = 200 * 1024;      // larger rows use the register kernel

template <int OP, bool PER_TOKEN, int CH>
fp8q_status launch_ring(const QuantParams& p, int T, cudaStream_t stream) {
  const int64_t row_bytes = (OP == OP_SILU ? 4 : 2) * p.L;
  const int stride = static_cast<int>(((row_bytes + 127) / 128) * 128);
  int nbuf = static_cast<int>(kRingSmemTarget / stride);
  nbuf = nbuf < 2 ? 2 : (nbuf > kRingMaxBuf ? kRingMaxBuf : nbuf);
  const int smem = nbuf * stride;
  auto kern = quant_ring_kernel<OP, PER_TOKEN, CH>;
  static int attr_done[64] = {0};
  static int occ_cache[64][2] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr_done[dev] = 1;
  }
  int occ = 0;
  if (occ_cache[dev][0] == (T << 20 | smem >> 7) + 1) {
    occ = occ_cache[dev][1];
  } else {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, T + 32, smem) != cudaSuccess || occ < 1)
      occ = 1;
    occ_cache[dev][0] = (T << 20 | smem >> 7) + 1;
    occ_cache[dev][1] = occ;
  }
  int64_t grid = static_cast<int64_t>(num_sms()) * occ;
  if (grid > p.M) grid = p.M;
  kern<<<static_cast<unsigned>(grid), T + 32, smem, stream>>>(p, nbuf, stride, device_status_ptr());
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
  // Long rows (8 chunks per thread, few rows per SM) stream through the
  // shared-memory ring; shorter rows run many CTAs per SM on registers alone.
  const int64_t row_bytes = (OP == OP_SILU ? 4 : 2) * p.L;
  if (ch == 8 && 2 * ((row_bytes + 127) / 128) * 128 <= kRingSmemMax)
    return per_token ? launch_ring<OP, true, 8>(p, T, stream) : launch_ring<OP, false, 8>(p, T, stream);
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
