// fp8q_quant.cu -- dynamic FP8 activation quantization fused with its producer.
//
// Ops ("Helion in vLLM" (24-ai.news), section "Kernels integrated into vLLM"):
//   items 1, 5  per-token / per-1x128-group quant          -> fp8q_group_quant
//   items 2, 6  RMSNorm + per-token / per-block quant       -> fp8q_rmsnorm_quant
//   items 3, 7  SiLU*mul + per-token / per-block quant      -> fp8q_silu_mul_quant
//
// One CTA (or, for long rows, one team of a CTA) owns one row.  Every thread
// loads its 16-byte chunks of the row (8 bf16 each; chunk c of the row goes
// to thread c mod T, so a warp reads 512 contiguous bytes per load), all loads
// issued before any arithmetic; many CTAs per SM keep enough loads in flight.
// The row then stays in registers as packed bf16 y values: one HBM read, one
// write of the codes.  Group amax = shuffle over the 16 threads that own one
// 128-wide group; row amax and the RMSNorm sum of squares = warp shuffle + a
// shared-memory pass over the warps.  Rows of more than 2048 chunks are
// streamed into shared memory by a bulk-copy ring instead (quant_ring_kernel).
//
// Exactness.  Codes and scales equal the definition bit for bit:
//   - the scale is fl32(max(amax, 1e-10) / 448) (IEEE division, recovered
//     from a product and its FMA residual); codes are the saturating RNE e4m3
//     of fl32(y / s), the IEEE quotient obtained with Markstein's division
//     step from the correctly rounded reciprocal of s (quant_chunk).
//   - y must be the correctly rounded bf16 of the op's real value.  RMSNorm:
//     n = bf16(x r) from a = rz(x r_lo) and b = rz(x r_hi) + 1 ulp, whose
//     magnitudes bracket |x r| for every x, subnormal results included;
//     SiLU*mul: the fp32 value and its proven error bound give the bracket.
//     Equal roundings of both ends are the rounding of the real value; pairs
//     whose ends differ (or, for SiLU, that are tiny or have a gate below
//     -85) are recomputed in fp64 and rounded to bf16 once.
//   - The RMSNorm sum of squares is accumulated in fp64, where squares of
//     bf16 values are exact; r is rsqrtf refined by one Newton step in fp64.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <atomic>

#include "fp8q_common.cuh"
#include "fp8q_quant_math.cuh"
#include "fp8q_sm100.cuh"

namespace fp8q {
namespace {

using namespace sm100;

// OP_ADD_RMS: residual add, then RMSNorm (h = bf16(x + residual) is written
// back to the residual and normalized).
enum { OP_PLAIN = 0, OP_RMS = 1, OP_SILU = 2, OP_ADD_RMS = 3 };
constexpr int kMaxThreads = 512;  // rows up to 8 * 8 * 512 = 32768 elements

struct QuantParams {
  const uint16_t* x;   // bf16 bits
  const uint16_t* w;   // bf16 bits (RMSNorm weight) or null
  float eps;
  int64_t M, L, ldx;   // L = row length of y (K, H or I)
  int group;           // 128 or L
  int ue8m0;           // 0 fp32 scales, 1 power-of-two fp32, 2 E8M0 bytes
  uint8_t* q;
  int64_t ldq;
  float* s;
  int64_t s_sm, s_sg;
  uint16_t* res;       // residual (bf16 bits, read and written) for OP_ADD_RMS
  int64_t ldr;
  int i8;              // 1: int8 codes, scale amax / 127 (W8A8_INT8)
};

// Store the scale of a group: fp32, or (ue8m0 = 2) its E8M0 byte -- the
// biased exponent of the power-of-two scale, which is a positive normal.
__device__ __forceinline__ void store_scale(const QuantParams& p, int64_t idx, float s) {
  if (p.ue8m0 == 2) reinterpret_cast<uint8_t*>(p.s)[idx] = static_cast<uint8_t>(__float_as_uint(s) >> 23);
  else p.s[idx] = s;
}

// Codes of a chunk in the format of the call.
__device__ __forceinline__ uint2 codes_chunk(const QuantParams& p, const uint4& y, const QScale& qs) {
  return p.i8 ? quant_chunk_i8(y, qs) : quant_chunk(y, qs);
}

// ---------------------------------------------------------------------------
// Kernels

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
// of 8 elements per thread; chunk c of the row belongs to thread c mod T, so
// every warp access is 512 contiguous bytes).  `release()` is called once the
// row's input has been read into registers.
// FAST (SiLU*mul): y from the fast arithmetic of the quant math header, then
// the elements within kCandSteps of their group's fast amax recomputed
// exactly before the scales are taken, so scales are exact and codes differ
// from the definition only where a fast y does.
template <int OP, bool PER_TOKEN, int CH, bool FAST, typename Src, typename Release>
__device__ __forceinline__ void process_row(const QuantParams& p, int64_t row, const Src& src,
                                            int tid, int T, int bar_id, double* red_d,
                                            float* red_f, Release release) {
  const int64_t nchunks = p.L >> 3;
  uint4 y[CH];
  bool valid[CH];
#pragma unroll
  for (int i = 0; i < CH; ++i) valid[i] = (tid + static_cast<int64_t>(i) * T) < nchunks;
  auto off = [&](int i) { return (tid + static_cast<int64_t>(i) * T) * 8; };
  // FAST: bit i set when chunk i holds an element whose fast |y| is within
  // kCandSteps bf16 steps of its group's fast amax (a team reduction per
  // token, four shuffles per 128-group).
  auto candidates = [&](const uint4* yy) {
    uint32_t cand = 0;
    if constexpr (PER_TOKEN) {
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < CH; ++i) m2 = chunk_absmax2(yy[i], m2);
      const float thr =
          bf16_steps_below(team_reduce(absmax2_to_f32(m2), MaxOp(), red_f, tid, T, bar_id), kCandSteps);
#pragma unroll
      for (int i = 0; i < CH; ++i)
        cand |= static_cast<uint32_t>(valid[i] && absmax2_to_f32(chunk_absmax2(yy[i], 0u)) >= thr) << i;
    } else {
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        const float a = absmax2_to_f32(chunk_absmax2(yy[i], 0u));
        float am = a;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
        cand |= static_cast<uint32_t>(valid[i] && a >= bf16_steps_below(am, kCandSteps)) << i;
      }
    }
    return cand;
  };

  // Hot loops compute every value on the fast path and only flag the rare
  // chunks with a pair whose rounding the fast path cannot decide; the exact
  // recomputation of those runs afterwards, outside the hot loops.
  uint32_t fix = 0;  // bit i: chunk i has a pair to recompute exactly
  if constexpr (OP == OP_PLAIN) {
#pragma unroll
    for (int i = 0; i < CH; ++i) y[i] = valid[i] ? src.ld(off(i)) : make_uint4(0, 0, 0, 0);
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
        if (valid[i0 + i] && FAST && chunk_min_gate(g[i]) >= -85.0f) {
          y[i0 + i].x = silu_pair_fast(g[i].x, u[i].x);
          y[i0 + i].y = silu_pair_fast(g[i].y, u[i].y);
          y[i0 + i].z = silu_pair_fast(g[i].z, u[i].z);
          y[i0 + i].w = silu_pair_fast(g[i].w, u[i].w);
        } else if (valid[i0 + i]) {
          uint32_t d = 0;
          bool bad = false;
          y[i0 + i].x = silu_pair(g[i].x, u[i].x, d, bad);
          y[i0 + i].y = silu_pair(g[i].y, u[i].y, d, bad);
          y[i0 + i].z = silu_pair(g[i].z, u[i].z, d, bad);
          y[i0 + i].w = silu_pair(g[i].w, u[i].w, d, bad);
          fix |= static_cast<uint32_t>(d != 0 || bad) << (i0 + i);
        } else {
          y[i0 + i] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    if (fix) {  // rare: re-read the flagged chunks and recompute them exactly
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if ((fix >> i) & 1u) y[i] = silu_chunk_fix(src.ld(off(i)), src.ld(p.L + off(i)), y[i]);
    }
    release();
  } else {  // OP_RMS, OP_ADD_RMS
    uint4 xv[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) xv[i] = valid[i] ? src.ld(off(i)) : make_uint4(0, 0, 0, 0);
    if constexpr (OP == OP_ADD_RMS) {
      // h = bf16(x + residual): the fp32 sum of two bf16 values is exact
      // unless their exponents are more than 16 apart, and then it lies far
      // from every bf16 rounding midpoint, so one RN to bf16 rounds the exact
      // sum.  h replaces the residual and is what gets normalized.
      uint16_t* rr = p.res + row * p.ldr;
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if (valid[i]) {
          const uint4 r = ld_stream(rr + off(i));
          uint4 h;
          h.x = f2_to_bf2_rn(add2(bf2_to_f2(xv[i].x), bf2_to_f2(r.x)));
          h.y = f2_to_bf2_rn(add2(bf2_to_f2(xv[i].y), bf2_to_f2(r.y)));
          h.z = f2_to_bf2_rn(add2(bf2_to_f2(xv[i].z), bf2_to_f2(r.z)));
          h.w = f2_to_bf2_rn(add2(bf2_to_f2(xv[i].w), bf2_to_f2(r.w)));
          *reinterpret_cast<uint4*>(rr + off(i)) = h;
          xv[i] = h;
        }
      }
    }
    release();
    // Sum of squares in fp64: squares of bf16 values are exact there (16
    // significant bits, exponents far inside the range).
    double a0 = 0.0, a1 = 0.0;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const double lo = __uint_as_float(xw[k] << 16), hi = __uint_as_float(xw[k] & 0xFFFF0000u);
        a0 = __fma_rn(lo, lo, a0);
        a1 = __fma_rn(hi, hi, a1);
      }
    }
    const double ss = team_reduce(a0 + a1, SumOp(), red_d, tid, T, bar_id);
    float r_lo, r_hi;
    rms_bracket(__fma_rn(ss, 1.0 / static_cast<double>(p.L), static_cast<double>(p.eps)), r_lo, r_hi);
    const uint64_t rlo2 = dup2(r_lo), rhi2 = dup2(r_hi);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if (valid[i]) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(p.w + off(i)));
        uint32_t d = 0;
        y[i].x = bf2_mul(rms_n_pair(xv[i].x, rlo2, rhi2, d), wv.x);
        y[i].y = bf2_mul(rms_n_pair(xv[i].y, rlo2, rhi2, d), wv.y);
        y[i].z = bf2_mul(rms_n_pair(xv[i].z, rlo2, rhi2, d), wv.z);
        y[i].w = bf2_mul(rms_n_pair(xv[i].w, rlo2, rhi2, d), wv.w);
        fix |= static_cast<uint32_t>(d != 0) << i;
      } else {
        y[i] = make_uint4(0, 0, 0, 0);
      }
    }
    if (fix) {  // rare: exact bf16(x r) for the pairs whose bracket is open
#pragma unroll
      for (int i = 0; i < CH; ++i)
        if ((fix >> i) & 1u)
          y[i] = rms_chunk_fix(xv[i], __ldg(reinterpret_cast<const uint4*>(p.w + off(i))), y[i], rlo2,
                               rhi2, ss, p.L, p.eps);
    }
  }
  if constexpr (FAST && OP == OP_SILU) {
    // The elements that can decide an amax, exactly (their gate and up
    // chunks read again from global memory).
    const uint32_t cand = candidates(y);
    const uint16_t* xr = p.x + row * p.ldx;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      if ((cand >> i) & 1u) {
        const uint4 g = ld_stream(xr + off(i)), u = ld_stream(xr + p.L + off(i));
        uint32_t d = 0;
        bool bad = false;
        y[i].x = silu_pair(g.x, u.x, d, bad);
        y[i].y = silu_pair(g.y, u.y, d, bad);
        y[i].z = silu_pair(g.z, u.z, d, bad);
        y[i].w = silu_pair(g.w, u.w, d, bad);
        if (d != 0 || bad) y[i] = silu_chunk_fix(g, u, y[i]);
      }
    }
  }

  uint8_t* qr = p.q + row * p.ldq;
  if constexpr (PER_TOKEN) {
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < CH; ++i) m2 = chunk_absmax2(y[i], m2);
    const float amax = team_reduce(absmax2_to_f32(m2), MaxOp(), red_f, tid, T, bar_id);
    const QScale qs = make_qscale(amax, p.ue8m0, p.i8);
#pragma unroll
    for (int i = 0; i < CH; ++i)
      if (valid[i]) *reinterpret_cast<uint2*>(qr + off(i)) = codes_chunk(p, y[i], qs);
    if (tid == 0) store_scale(p, row * p.s_sm, qs.s);
  } else {
    // 128-wide groups: the 16 threads tid & ~15 .. +15 own one group per i
    // (T is a multiple of 32 and L of 128, so whole half-warps are valid or not).
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      float a = absmax2_to_f32(chunk_absmax2(y[i], 0u));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      if (valid[i]) {
        const QScale qs = make_qscale(a, p.ue8m0, p.i8);
        *reinterpret_cast<uint2*>(qr + off(i)) = codes_chunk(p, y[i], qs);
        if ((tid & 15) == 0) store_scale(p, row * p.s_sm + (off(i) >> 7) * p.s_sg, qs.s);
      }
    }
  }
}

// Register kernel: one CTA per row, the row loaded straight into registers.
// Used for rows too long for the shared-memory ring below.
// MAXT/MINB set the register budget (measured): 64 registers for 4 chunks
// per thread (plain and RMSNorm: the occupancy beats the few spills), 80 for
// SiLU rows of up to 384 threads, 128 for 8 chunks per thread.
template <int OP, bool PER_TOKEN, int CH, int MAXT, int MINB, bool FAST>
__global__ void __launch_bounds__(MAXT, MINB) quant_rows_kernel(const QuantParams p) {
  __shared__ double red_d[32];
  __shared__ float red_f[32];
  griddep_wait();                 // x (and w) may come from the previous kernel
  griddep_launch_dependents();
  for (int64_t row = blockIdx.x; row < p.M; row += gridDim.x)
    process_row<OP, PER_TOKEN, CH, FAST>(p, row, GlobalRow{p.x + row * p.ldx}, threadIdx.x, blockDim.x,
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
  return ch == 8 ? 512 : (op == OP_SILU ? 800 : (op == OP_ADD_RMS ? 768 : 1024));
}

template <int OP, bool PER_TOKEN, int CH, bool FAST>
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
  griddep_wait();                 // x may come from the previous kernel
  griddep_launch_dependents();

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
    process_row<OP, PER_TOKEN, CH, FAST>(p, row, SmemRow{src}, tid, T, bar, red_d[team], red_f[team], [&] {
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

constexpr int kRingSmemMax = 216 * 1024;   // ring bytes per CTA (one CTA per SM; 2 slots of a
                                           // 25600-wide SiLU row fit)

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

template <int OP, bool PER_TOKEN, int CH, bool FAST>
fp8q_status launch_ring(const QuantParams& p, int T, int nteams, int nbuf, int stride,
                        cudaStream_t stream) {
  const int smem = nbuf * stride;
  auto kern = quant_ring_kernel<OP, PER_TOKEN, CH, FAST>;
  static std::atomic<int> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  if (!attr_done[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr_done[dev].store(1, std::memory_order_relaxed);
  }
  int64_t grid = num_sms();
  if (grid > p.M) grid = p.M;
  return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(32 + nteams * T), smem, stream,
                       1, p, nbuf, nteams, T, stride, device_status_ptr());
}

// Staged SiLU*mul per-token kernel (long rows): persistent CTAs, one row at
// a time per CTA.  Warp 0 (one lane) streams whole [gate | up] rows into NBUF
// slots of shared memory with cp.async.bulk, as in the ring kernel; the other T
// threads all work on the same row (chunk c to thread c mod T, at most
// kStagedPasses chunks a thread).  Phase 1 turns each chunk of gate and up into
// y = bf16(silu(g) u), stores y over the chunk's gate bytes and keeps the
// thread's amax; one CTA-wide reduction gives the row's scale; phase 2 reads
// the y chunks back and writes the codes.  y never stays in registers across
// the row reduction, so a row of 25600 values is worked on by up to 992
// threads instead of the ~400 that a register-resident row fits.  FAST: the
// chunks holding an element within kCandSteps of the fast amax are recomputed
// exactly (gate and up read again from global memory) and the amax reduced
// again.  Slots go back to the producer after a proxy fence (the y stores are
// generic writes to bytes the next bulk copy overwrites).  Waits are bounded
// as in the ring kernel.
constexpr int kStagedMaxThreads = 1024;
constexpr int kStagedPasses = 4;

// max of two packed pairs of bf16 magnitudes
__device__ __forceinline__ uint32_t absmax2_merge(uint32_t a, uint32_t b) {
  const __nv_bfloat162 m = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                   *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<const uint32_t*>(&m);
}

template <bool FAST>
__global__ void __launch_bounds__(kStagedMaxThreads, 1)
    silu_staged_kernel(const QuantParams p, int nbuf, int T, int row_stride_bytes, int* status) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kRingMaxBuf], empty[kRingMaxBuf];
  __shared__ float red_f[32];
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t copy_bytes = static_cast<uint32_t>(4 * p.L);
  const int64_t nchunks = p.L >> 3;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nbuf; ++i) {
      sm100::mbar_init(&full[i], 1);
      sm100::mbar_init(&empty[i], T / 32);
    }
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();                 // x may come from the previous kernel
  griddep_launch_dependents();

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
  constexpr int bar = 1;
  int i = 0;
  for (int64_t row = blockIdx.x; row < p.M; row += gridDim.x, ++i) {
    const int slot = i % nbuf;
    const bool ok = sm100::mbar_wait(&full[slot], (i / nbuf) & 1, &abort_flag, status);
    if (sm100::team_any(!ok, bar, T)) break;
    uint8_t* base = ring + static_cast<size_t>(slot) * row_stride_bytes;
    uint8_t* qr = p.q + row * p.ldq;
    auto exact_chunk = [](const uint4& g, const uint4& u) {
      uint32_t d = 0;
      bool bad = false;
      uint4 y;
      y.x = silu_pair(g.x, u.x, d, bad);
      y.y = silu_pair(g.y, u.y, d, bad);
      y.z = silu_pair(g.z, u.z, d, bad);
      y.w = silu_pair(g.w, u.w, d, bad);
      if (d != 0 || bad) y = silu_chunk_fix(g, u, y);   // rare: exact recomputation
      return y;
    };
    uint32_t cm[kStagedPasses];      // packed absmax of each of this thread's chunks
    uint32_t m2 = 0;
#pragma unroll
    for (int k = 0; k < kStagedPasses; ++k) {
      const int64_t c = tid + static_cast<int64_t>(k) * T;
      cm[k] = 0;
      if (c < nchunks) {
        const uint4 g = *reinterpret_cast<const uint4*>(base + 16 * c);
        const uint4 u = *reinterpret_cast<const uint4*>(base + 2 * p.L + 16 * c);
        uint4 y;
        if (FAST && chunk_min_gate(g) >= -85.0f) {
          y.x = silu_pair_fast(g.x, u.x);
          y.y = silu_pair_fast(g.y, u.y);
          y.z = silu_pair_fast(g.z, u.z);
          y.w = silu_pair_fast(g.w, u.w);
        } else {
          y = exact_chunk(g, u);
        }
        cm[k] = chunk_absmax2(y, 0u);
        m2 = absmax2_merge(m2, cm[k]);
        *reinterpret_cast<uint4*>(base + 16 * c) = y;
      }
    }
    float amax = team_reduce(absmax2_to_f32(m2), MaxOp(), red_f, tid, T, bar);
    if constexpr (FAST) {
      const float thr = bf16_steps_below(amax, kCandSteps);
      const uint16_t* xr = p.x + row * p.ldx;
      m2 = 0;
#pragma unroll
      for (int k = 0; k < kStagedPasses; ++k) {
        const int64_t c = tid + static_cast<int64_t>(k) * T;
        if (c < nchunks && absmax2_to_f32(cm[k]) >= thr) {
          const uint4 y = exact_chunk(ld_stream(xr + 8 * c), ld_stream(xr + p.L + 8 * c));
          cm[k] = chunk_absmax2(y, 0u);
          *reinterpret_cast<uint4*>(base + 16 * c) = y;
        }
        m2 = absmax2_merge(m2, cm[k]);
      }
      amax = team_reduce(absmax2_to_f32(m2), MaxOp(), red_f, tid, T, bar);
    }
    const QScale qs = make_qscale(amax, p.ue8m0, p.i8);
#pragma unroll
    for (int k = 0; k < kStagedPasses; ++k) {
      const int64_t c = tid + static_cast<int64_t>(k) * T;
      if (c < nchunks)
        *reinterpret_cast<uint2*>(qr + 8 * c) = codes_chunk(p, *reinterpret_cast<const uint4*>(base + 16 * c), qs);
    }
    if (tid == 0) store_scale(p, row * p.s_sm, qs.s);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty[slot]);
  }
}

// Staged-kernel geometry for a row of L values: T = the fewest threads (a
// multiple of 32, at most 992) that cover the row's chunks in the fewest
// passes, and as many row slots (at most 16) as fit the shared memory.  False
// when fewer than two slots fit.
bool staged_geometry(int64_t L, int* T, int* nbuf, int* stride) {
  const int64_t nchunks = L >> 3;
  const int64_t tmax = kStagedMaxThreads - 32;
  const int64_t passes = (nchunks + tmax - 1) / tmax;
  if (passes > kStagedPasses) return false;
  const int64_t t = ((nchunks + passes - 1) / passes + 31) / 32 * 32;
  const int64_t st = (4 * L + 127) / 128 * 128;
  if (st * 2 > kRingSmemMax) return false;
  int64_t nb = kRingSmemMax / st;
  if (nb > kRingMaxBuf) nb = kRingMaxBuf;
  *T = static_cast<int>(t);
  *nbuf = static_cast<int>(nb);
  *stride = static_cast<int>(st);
  return true;
}

template <bool FAST>
fp8q_status launch_staged(const QuantParams& p, int T, int nbuf, int stride, cudaStream_t stream) {
  auto kern = silu_staged_kernel<FAST>;
  static std::atomic<int> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return FP8Q_ERR_CUDA;
  if (!attr_done[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr_done[dev].store(1, std::memory_order_relaxed);
  }
  int64_t grid = num_sms();
  if (grid > p.M) grid = p.M;
  return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(32 + T), nbuf * stride, stream, 1, p,
                       nbuf, T, stride, device_status_ptr());
}

// Group kernel: 1x128 groups of the SiLU*mul quant, which need no row-wide
// value, as independent items.  Item i = (row i / G, group
// i % G); a team of 16 consecutive threads owns one item, 8 elements (one
// 16-byte chunk of x, or of gate and of up) per thread, so a warp reads two
// groups' 256 contiguous bytes per load; every thread keeps kGroupItems items
// in flight (all loads issued before any arithmetic).  The group amax is four
// shuffles inside the team; codes and scales are exactly those of the row
// kernels (same helpers, same exactness).  No block barriers.
constexpr int kGroupThreads = 256;
constexpr int kGroupItems = 4;

template <int OP>
__global__ void __launch_bounds__(kGroupThreads) quant_groups_kernel(const QuantParams p) {
  constexpr int TEAMS = kGroupThreads / 16;
  const int t = threadIdx.x & 15;
  const int team = threadIdx.x >> 4;
  const int64_t G = p.L >> 7;
  const int64_t items = p.M * G;
  griddep_wait();                 // x may come from the previous kernel
  griddep_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * TEAMS * kGroupItems;
  // item -> row: a 32-bit division whenever the item count allows it (a
  // 64-bit one is a long software sequence, paid once per 8 elements)
  const bool narrow = items <= 0xFFFFFFFFll;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * TEAMS * kGroupItems; base < items;
       base += stride) {
    int64_t row[kGroupItems], col[kGroupItems];
    bool ok[kGroupItems];
    uint4 a[kGroupItems], b[kGroupItems];
#pragma unroll
    for (int u = 0; u < kGroupItems; ++u) {
      const int64_t it = base + team + static_cast<int64_t>(u) * TEAMS;
      ok[u] = it < items;
      row[u] = !ok[u] ? 0
               : narrow ? static_cast<int64_t>(static_cast<uint32_t>(it) / static_cast<uint32_t>(G))
                        : it / G;
      col[u] = ok[u] ? (it - row[u] * G) * 128 + 8 * t : 0;      // element offset in the row
      const uint16_t* xr = p.x + row[u] * p.ldx;
      a[u] = ok[u] ? ld_stream(xr + col[u]) : make_uint4(0, 0, 0, 0);
      if constexpr (OP == OP_SILU) b[u] = ok[u] ? ld_stream(xr + p.L + col[u]) : make_uint4(0, 0, 0, 0);
      else b[u] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kGroupItems; ++u) {
      uint4 y;
      if constexpr (OP == OP_SILU) {
        uint32_t d = 0;
        bool bad = false;
        y.x = silu_pair(a[u].x, b[u].x, d, bad);
        y.y = silu_pair(a[u].y, b[u].y, d, bad);
        y.z = silu_pair(a[u].z, b[u].z, d, bad);
        y.w = silu_pair(a[u].w, b[u].w, d, bad);
        if (d != 0 || bad) y = silu_chunk_fix(a[u], b[u], y);   // rare: exact recomputation
      } else {
        y = a[u];
      }
      float am = absmax2_to_f32(chunk_absmax2(y, 0u));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
      const QScale qs = make_qscale(am, p.ue8m0, p.i8);
      if (ok[u]) {
        *reinterpret_cast<uint2*>(p.q + row[u] * p.ldq + col[u]) = codes_chunk(p, y, qs);
        if (t == 0) store_scale(p, row[u] * p.s_sm + (col[u] >> 7) * p.s_sg, qs.s);
      }
    }
  }
}

template <int OP, bool FAST>
fp8q_status launch_quant_mode(const QuantParams& p, cudaStream_t stream) {
  if (p.M == 0) return FP8Q_OK;
  const int64_t nchunks = p.L / 8;
  const bool per_token = p.group == p.L;
  if constexpr (OP == OP_SILU) {
    // Long per-token rows (more than 2048 chunks): the staged kernel
    // (measured at I = 25600: 399 us against 514 for the ring kernel; at
    // I = 12288 the register kernel stays faster, 190 against 274 us).
    int T = 0, nbuf = 0, stride = 0;
    if (per_token && nchunks > 2048 && staged_geometry(p.L, &T, &nbuf, &stride))
      return launch_staged<FAST>(p, T, nbuf, stride, stream);
    if (!per_token) {
      // 1x128 groups: independent items, no row-wide reduction (measured:
      // faster than the row kernels for SiLU*mul; for the plain quant the
      // row kernel is faster)
      constexpr int64_t per_block = (kGroupThreads / 16) * kGroupItems;
      const int64_t items = p.M * (p.L >> 7);
      int64_t blocks = (items + per_block - 1) / per_block;
      const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
      if (blocks > cap) blocks = cap;
      return launch_kernel(quant_groups_kernel<OP>, dim3(static_cast<unsigned>(blocks)),
                           dim3(kGroupThreads), 0, stream, 1, p);
    }
  }
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
    return per_token ? launch_ring<OP, true, 8, FAST>(p, T, nteams, nbuf, stride, stream)
                     : launch_ring<OP, false, 8, FAST>(p, T, nteams, nbuf, stride, stream);
  const int64_t grid = p.M < (1LL << 30) ? p.M : (1LL << 30);
  const dim3 g(static_cast<unsigned>(grid)), b(T);
  auto go = [&](auto kern) { return launch_kernel(kern, g, b, 0, stream, 1, p); };
  if (ch == 8)
    return per_token ? go(quant_rows_kernel<OP, true, 8, 512, 1, FAST>) : go(quant_rows_kernel<OP, false, 8, 512, 1, FAST>);
  // residual add + RMSNorm rows of up to 256 threads: five CTAs per SM (48
  // registers, some spilled) measured 6-7% faster than four at H = 4096 and
  // 5120; the plain RMSNorm rows measured slower that way
  if (OP == OP_ADD_RMS && T <= 256)
    return per_token ? go(quant_rows_kernel<OP, true, 4, 256, 5, FAST>) : go(quant_rows_kernel<OP, false, 4, 256, 5, FAST>);
  if (OP == OP_SILU && T <= 256)
    return per_token ? go(quant_rows_kernel<OP, true, 4, 256, 3, FAST>) : go(quant_rows_kernel<OP, false, 4, 256, 3, FAST>);
  if (OP == OP_SILU && T <= 384)
    return per_token ? go(quant_rows_kernel<OP, true, 4, 384, 2, FAST>) : go(quant_rows_kernel<OP, false, 4, 384, 2, FAST>);
  return per_token ? go(quant_rows_kernel<OP, true, 4, 512, 2, FAST>) : go(quant_rows_kernel<OP, false, 4, 512, 2, FAST>);
}

// SiLU*mul per token runs its fast y unless the exact mode is set
// (fp8q_set_fused_quant_exact).  Everything else is exact in both modes: the
// plain quant by definition; RMSNorm (row kernels, ring), residual add +
// RMSNorm and the 1x128 SiLU*mul kernel measured no faster with the fast
// arithmetic (their time goes to row latency and to the extra amax pass).
std::atomic<int> g_fused_exact{0};

template <int OP>
fp8q_status launch_quant(const QuantParams& p, cudaStream_t stream) {
  if constexpr (OP != OP_SILU) {
    return launch_quant_mode<OP, false>(p, stream);
  } else {
    return g_fused_exact.load(std::memory_order_relaxed) ? launch_quant_mode<OP, false>(p, stream)
                                                         : launch_quant_mode<OP, true>(p, stream);
  }
}

// Host-side validation shared by the three ops (row length L of y).
fp8q_status check_common(const void* x, int64_t M, int64_t L, int64_t ldx, int64_t ld_in_min,
                         int group, int ue8m0, const void* q, int64_t ldq, const float* s,
                         int64_t s_sm, int64_t s_sg) {
  if (M < 0 || L <= 0 || L % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (ldx < ld_in_min || ldx % 8 != 0 || ldq < L || ldq % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (!(group == 128 && L % 128 == 0) && static_cast<int64_t>(group) != L) return FP8Q_ERR_INVALID_ARG;
  if (ue8m0 < 0 || ue8m0 > 2) return FP8Q_ERR_INVALID_ARG;
  if (s_sm < 0 || s_sg < 0) return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;  // nothing is read or written: pointers may be null
  if (!x || !q || !s) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s, ue8m0 == 2 ? 1 : 4)) return FP8Q_ERR_INVALID_ARG;
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

extern "C" fp8q_status fp8q_add_rmsnorm_quant(const void* x, void* residual, const void* w, float eps,
                                              int64_t M, int64_t H, int64_t ldx, int64_t ldr,
                                              int group_size, int ue8m0, void* q, int64_t ldq,
                                              float* scales, int64_t s_stride_m, int64_t s_stride_g,
                                              void* stream) {
  fp8q_status st = check_common(x, M, H, ldx, H, group_size, ue8m0, q, ldq, scales, s_stride_m,
                                s_stride_g);
  if (st != FP8Q_OK) return st;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return FP8Q_ERR_INVALID_ARG;
  if (ldr < H || ldr % 8 != 0) return FP8Q_ERR_INVALID_ARG;
  if (M > 0 && (!w || !aligned(w, 16) || !residual || !aligned(residual, 16))) return FP8Q_ERR_INVALID_ARG;
  QuantParams p{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w), eps, M, H, ldx,
                group_size, ue8m0, static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g,
                static_cast<uint16_t*>(residual), ldr};
  return launch_quant<OP_ADD_RMS>(p, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- W8A8_INT8
// The same three producers with int8 codes (scale amax / 127).
extern "C" fp8q_status fp8q_group_quant_i8(const void* x, int64_t M, int64_t K, int64_t ldx,
                                           int group_size, void* q, int64_t ldq, float* scales,
                                           int64_t s_stride_m, int64_t s_stride_g, void* stream) {
  fp8q_status st = check_common(x, M, K, ldx, K, group_size, 0, q, ldq, scales, s_stride_m,
                                s_stride_g);
  if (st != FP8Q_OK) return st;
  QuantParams p{static_cast<const uint16_t*>(x), nullptr, 0.0f, M, K, ldx, group_size, 0,
                static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g, nullptr, 0, 1};
  return launch_quant<OP_PLAIN>(p, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_rmsnorm_quant_i8(const void* x, const void* w, float eps, int64_t M,
                                             int64_t H, int64_t ldx, int group_size, void* q,
                                             int64_t ldq, float* scales, int64_t s_stride_m,
                                             int64_t s_stride_g, void* stream) {
  fp8q_status st = check_common(x, M, H, ldx, H, group_size, 0, q, ldq, scales, s_stride_m,
                                s_stride_g);
  if (st != FP8Q_OK) return st;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return FP8Q_ERR_INVALID_ARG;
  if (M > 0 && (!w || !aligned(w, 16))) return FP8Q_ERR_INVALID_ARG;
  QuantParams p{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(w), eps, M, H, ldx,
                group_size, 0, static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g, nullptr,
                0, 1};
  return launch_quant<OP_RMS>(p, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_silu_mul_quant_i8(const void* x, int64_t M, int64_t I, int64_t ldx,
                                              int group_size, void* q, int64_t ldq, float* scales,
                                              int64_t s_stride_m, int64_t s_stride_g, void* stream) {
  if (I > (INT64_MAX / 4)) return FP8Q_ERR_INVALID_ARG;
  fp8q_status st = check_common(x, M, I, ldx, 2 * I, group_size, 0, q, ldq, scales, s_stride_m,
                                s_stride_g);
  if (st != FP8Q_OK) return st;
  QuantParams p{static_cast<const uint16_t*>(x), nullptr, 0.0f, M, I, ldx, group_size, 0,
                static_cast<uint8_t*>(q), ldq, scales, s_stride_m, s_stride_g, nullptr, 0, 1};
  return launch_quant<OP_SILU>(p, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_set_fused_quant_exact(int exact) {
  if (exact != 0 && exact != 1) return FP8Q_ERR_INVALID_ARG;
  g_fused_exact.store(exact, std::memory_order_relaxed);
  return FP8Q_OK;
}

extern "C" int fp8q_get_fused_quant_exact(void) { return g_fused_exact.load(std::memory_order_relaxed); }
