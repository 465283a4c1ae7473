// fp8q_gemm.cu -- scaled FP8 GEMMs on the 5th-generation tensor cores (sm_100a).
//
//   scaled_mm            y = bf16(sa(m) sb(n) sum_k qa[m,k] qb[n,k])
//   scaled_mm_blockwise  y = bf16(sum_kb sa[m,kb] sb[n/128,kb] P_kb[m,n])
// ("Helion in vLLM" (24-ai.news), section "Kernels integrated into vLLM",
// items 8 and 9; the FP8_Dynamic and Block_FP8 schemes of "Helion linear
// backend" (aihirek.info), section "Autotuning selects the variant").
//
// One persistent kernel template, one CTA per SM, warp-specialized:
//   warp 0      TMA producer: 128-row x 128-byte e4m3 tiles of both operands,
//               128B-swizzled, into a STAGES-deep shared-memory ring guarded
//               by full/empty mbarriers;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//               (kind::f8f6f4, M = 128, N = BN, K = 32 per instruction);
//   warps 2..   epilogue: tcgen05.ld of the fp32 accumulator, scales, bf16.
// Per-token/per-channel scales: the accumulator of a whole tile lives in one
// of two TMEM buffers, so the epilogue of tile t overlaps the mainloop of
// tile t+1.  Blockwise scales: each 128-deep K block accumulates into its own
// TMEM partial buffer (4 rotating buffers); the epilogue promotes every partial
// into fp32 registers with its scale sa[m,kb]*sb[nb,kb].
//
// Variants ("Helion linear backend" (aihirek.info), section "Single GEMM
// implementation handles several algorithms"):
//   Swap-AB  the weight rows fill the MMA's 128-row M slot and the tokens its
//            N slot (BN = 16..128), for small M;
//   Split-K  the K loop of a tile is cut into `split` ranges run by different
//            CTAs; each writes a scaled fp32 partial to the workspace and the
//            last one to arrive (per-warp atomic counter) sums the partials in
//            split order (deterministic) and writes y.
// No TMA multicast is used: every CTA loads its own tiles.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>
#include <mutex>
#include <unordered_map>

#include "fp8q_common.cuh"
#include "fp8q_quant_math.cuh"
#include "fp8q_sm100.cuh"

namespace fp8q {
namespace {

using namespace sm100;

constexpr int BM = 128;       // MMA M = TMEM lanes per tile
constexpr int BK = 128;       // K bytes (e4m3 elements) per pipeline stage
constexpr int UMMA_K = 32;    // K per tcgen05.mma for 8-bit operands
constexpr int A_BYTES = BM * BK;
constexpr int kSmemBudget = 200 * 1024;

// Register split of the blockwise 128x256 kernel (setmaxnreg): its 8
// epilogue warps hold 128 fp32 accumulators a thread, which leaves no room for
// wide TMEM loads at the 168 registers a thread of a 10-warp CTA.  With the
// split the CTA has 12 warps -- epilogue warps 0-7 (two warpgroups), the TMA
// producer warp 8, the MMA warp 9, two idle -- and after setup the third
// warpgroup drops to kRegLow registers while the epilogue warpgroups rise
// to kRegHigh.  The sum 256 kRegHigh + 128 kRegLow = 60416 stays below the
// CTA's allocation at launch even at 160 registers a thread (61440), so the
// raise never waits.
#ifndef FP8Q_REGSPLIT
#define FP8Q_REGSPLIT 0
#endif
constexpr bool kRegSplit = FP8Q_REGSPLIT != 0;
constexpr int kRegLow = 40, kRegHigh = 216;
static_assert(256 * kRegHigh + 128 * kRegLow <= 384 * 160, "register split exceeds the launch allocation");

// Test-only build switch (-DFP8Q_TEST_STALL_PRODUCER=1, never in the shipped
// library): the GEMM's TMA producer issues nothing, so the MMA thread's first
// pipeline wait runs out and the kernel takes its timeout path (abort flag,
// FP8Q_ERR_TIMEOUT in the status word, drain, TMEM release, return).
#ifdef FP8Q_TEST_STALL_PRODUCER
constexpr bool kTestStallProducer = FP8Q_TEST_STALL_PRODUCER != 0;
#else
constexpr bool kTestStallProducer = false;
#endif

struct GemmArgs {
  int rows_a, rows_b, K;              // MMA-A rows (TMEM lanes), MMA-B rows (columns)
  int kblocks, tiles_a, tiles_b, split, kb_per_split, units;  // classic: tiles x split units
  int streamk;                        // 1: stream-K ranges instead of units
  int seg_len, total_iters;           // stream-K: K-block iterations per CTA, tiles x kblocks
  int max_contrib;                    // partial slots per tile in the workspace
  int M, N;                           // logical output shape
  const float* sa;                    // activation scales: sa[m*sa_sm + kb*sa_skb]
  int64_t sa_sm, sa_skb;
  const float* sb;                    // weight scales: per channel sb[n*sb_sn];
  int64_t sb_sn, sb_snb, sb_skb;      //   blockwise sb[(n/128)*sb_snb + kb*sb_skb]
  uint16_t* y;                        // bf16 [M, ldy]
  int64_t ldy;
  float* ws;                          // split-K partials
  int* counters;                      // split-K arrival counters (zero between calls)
  int* status;                        // device status word
  // E8M0 block scales (block-scaled MMA): activations sfa[m*sfa_sm + kb*sfa_skb],
  // weights sfb[(n/128)*sfb_snb + kb]
  const uint8_t* sfa;
  int64_t sfa_sm, sfa_skb;
  const uint8_t* sfb;
  int64_t sfb_snb;
  // SiLU*mul quant fused into the epilogue (gate_up): codes q[m*sq_ldq + o],
  // scale of group (m, o/128) at sq_s[m*sq_s_sm + (o/128)*sq_s_sg] (fp32, or
  // an E8M0 byte when sq_ue8m0 = 2)
  uint8_t* sq_q;
  int64_t sq_ldq;
  float* sq_s;
  int64_t sq_s_sm, sq_s_sg;
  int sq_ue8m0;
  // 1: every SiLU*mul value exact; 0 (fast): an open pair is kept within one
  // bf16 step of its value unless its chunk can decide the group amax
  int sq_exact;
};

// MX: E8M0 block scales applied by the tensor core (kind::mxf8f6f4.block_scale);
// the accumulator then needs no scaling, as with unit per-token scales.
// I8: W8A8_INT8, signed 8-bit operands (kind::i8) with s32 accumulators and
// per-token / per-channel scales.
template <int BN, bool SWAP, bool BW, bool MX = false, bool I8 = false>
struct Cfg {
  static_assert(!(BW && MX) && !(I8 && (BW || MX)), "one scale scheme");
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;           // TMA bytes per stage
  // Scale factors (MX): per pipeline stage a shared-memory slot of 512 bytes
  // for the 128 MMA rows and 512 per 128 MMA columns, written by the SF warp,
  // and a TMEM slot of 4 + 4 per 128 columns, filled from it by the MMA
  // thread with tcgen05.cp.
  static constexpr int SFB_CHUNKS = (BN + 127) / 128;
  static constexpr int SF_COLS = 4 * (1 + SFB_CHUNKS);
  static constexpr int SF_BYTES = MX ? 512 * (1 + SFB_CHUNKS) : 0;
  static constexpr int SF_WARPS = MX ? 1 : 0;
  static constexpr int STAGES_RAW = kSmemBudget / (STAGE_BYTES + SF_BYTES);
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int EPI_WARPS = (BW && BN >= 128) ? 8 : 4;
  static constexpr int COL_GROUPS = EPI_WARPS / 4;        // column slices per TMEM lane quadrant
  static constexpr int CPT = BN / COL_GROUPS;              // columns per epilogue thread
  // Columns per tcgen05.ld.  The blockwise epilogue keeps two chunks in
  // flight (the next one loads while the current one is scaled); its
  // 256-column tile holds 128 fp32 accumulators per thread (8 epilogue warps,
  // 10 in all: 168 registers a thread), so it reads 8 columns at a time.
  static constexpr int CHUNK = BW ? (CPT >= 128 ? (kRegSplit && BN == 256 && !SWAP ? 32 : 8) : 16)
                                  : (CPT < 32 ? 16 : 32);
  // TMEM accumulator buffers.  The E8M0 kernel's 256-column tile keeps one
  // (two would leave no columns for the scale factors): its tile epilogue is
  // not overlapped with the next tile's MMAs, and still measured 5-8% faster
  // than 224-column tiles with two buffers, the block-scaled MMA's cost per
  // instruction being spread over more columns.
  static constexpr int NBUF = (MX && BN == 256) ? 1 : (BW && BN < 256) ? 4 : 2;
  static constexpr int SF_COL0 = NBUF * BN;                 // first scale-factor column (MX)
  static constexpr int TMEM_NEED = NBUF * BN + (MX ? STAGES * SF_COLS : 0);
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64
                                 : TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  // register split: see kRegSplit (blockwise 128x256 tiles only)
  static constexpr bool REGSPLIT = kRegSplit && BW && BN == 256 && !SWAP;
  static constexpr int W_PROD = REGSPLIT ? EPI_WARPS : 0;       // TMA producer warp
  static constexpr int W_MMA = REGSPLIT ? EPI_WARPS + 1 : 1;    // TMEM allocator and MMA warp
  static constexpr int EPI_BASE = REGSPLIT ? 0 : 2;             // first epilogue warp
  static constexpr int THREADS = REGSPLIT ? 384 : 64 + 32 * (EPI_WARPS + SF_WARPS);
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * NBUF + 1) + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * (STAGE_BYTES + SF_BYTES) + BAR_BYTES;
  static_assert(STAGES >= 2, "pipeline too shallow");
  static_assert(TMEM_NEED <= 512, "accumulators exceed TMEM");
  static_assert(CPT % CHUNK == 0 && (CHUNK == 8 || CHUNK == 16 || CHUNK == 32), "chunking");
  static_assert(B_BYTES % 1024 == 0, "B tiles must stay 1024-byte aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void unit_coords(const GemmArgs& p, int u, int& ta, int& tb, int& s,
                                            int& kb0, int& kb1) {
  ta = u % p.tiles_a;
  const int r = u / p.tiles_a;
  tb = r % p.tiles_b;
  s = r / p.tiles_b;
  kb0 = s * p.kb_per_split;
  kb1 = min(p.kblocks, kb0 + p.kb_per_split);
}

// One piece of work of a CTA: K blocks [kb0, kb1) of tile (ta, tb), written
// to partial slot `slot` of the tile's `ncontrib` contributors (1: the piece
// is the whole tile and goes straight to y).
struct Seg {
  int ta, tb, kb0, kb1, slot, ncontrib;
};

// The CTA's pieces in order.  Classic: units blockIdx.x, + gridDim.x, ...
// (tile-major, `split` equal K ranges per tile).  Stream-K: one contiguous
// range of seg_len (tile, K block) iterations per CTA, so every CTA streams
// the same number of K blocks; a tile cut by range boundaries is summed from
// the partials of the CTAs that cover it, in CTA order.
struct SegIter {
  int cur, end;
  __device__ explicit SegIter(const GemmArgs& p) {
    if (p.streamk) {
      cur = blockIdx.x * p.seg_len;
      end = min(p.total_iters, cur + p.seg_len);
    } else {
      cur = blockIdx.x;
      end = p.units;
    }
  }
  __device__ bool next(const GemmArgs& p, Seg& g) {
    if (cur >= end) return false;
    if (!p.streamk) {
      unit_coords(p, cur, g.ta, g.tb, g.slot, g.kb0, g.kb1);
      g.ncontrib = p.split;
      cur += gridDim.x;
      return true;
    }
    const int tile = cur / p.kblocks;
    g.kb0 = cur - tile * p.kblocks;
    g.kb1 = min(p.kblocks, g.kb0 + (end - cur));
    g.ta = tile % p.tiles_a;
    g.tb = tile / p.tiles_a;
    const int first = static_cast<int>((static_cast<int64_t>(tile) * p.kblocks) / p.seg_len);
    const int last = static_cast<int>((static_cast<int64_t>(tile + 1) * p.kblocks - 1) / p.seg_len);
    g.ncontrib = last - first + 1;
    g.slot = static_cast<int>(blockIdx.x) - first;
    cur += g.kb1 - g.kb0;
    return true;
  }
};

// acc += (r0, r1) * sc: one paired fp32 FMA (sm_100 .f32x2) on a 64-bit
// accumulator pair; r0, r1 are adjacent registers of a tcgen05.ld.
__device__ __forceinline__ void ffma2_acc(uint64_t& acc, uint32_t r0, uint32_t r1, uint64_t sc) {
  asm("{\n\t.reg .b64 v;\n\t"
      "mov.b64 v, {%1, %2};\n\t"
      "fma.rn.f32x2 %0, v, %3, %0;\n\t}"
      : "+l"(acc)
      : "r"(r0), "r"(r1), "l"(sc));
}

__device__ __forceinline__ uint64_t pair_f32(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpair_f32(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// SQ (blockwise, 128x256 tiles, no swap, whole K): the gate_up GEMM with the
// SiLU*mul quant in its epilogue.  The weight rows come interleaved in
// 128-row blocks, [gate block j | up block j] for j = 0, 1, ..., so tile tb
// holds gate outputs [128 tb, 128 tb + 128) in columns 0-127 and the matching
// up outputs in columns 128-255.  Each epilogue thread owns 64 gate and the
// matching 64 up columns of its row; after the K loop it rounds both to bf16
// as the GEMM emits them, applies the SiLU*mul of the quant kernels (exact,
// or in the fast mode exact wherever a value can decide the group amax),
// takes the 1x128 group amax with its partner thread (the other column
// slice, same row) through shared memory and writes e4m3 codes and the
// group's scale.  The 2I-wide bf16 intermediate is never written.
template <int BN, bool SWAP, bool BW, bool MX, bool I8, bool SQ>
__global__ void __launch_bounds__(Cfg<BN, SWAP, BW, MX, I8>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs p) {
  using C = Cfg<BN, SWAP, BW, MX, I8>;
  static_assert(!SQ || (BW && !SWAP && BN == 256 && C::EPI_WARPS == 8 && 64 % C::CHUNK == 0),
                "the fused SiLU*mul quant epilogue runs on 128x256 blockwise tiles");
  // SQ: per-slice partial group amax, double-buffered by tile parity, and one
  // mbarrier per TMEM lane quadrant (one arrival from each of its two warps,
  // which hold the two column slices of the same rows, per tile)
  __shared__ float sq_red[SQ ? 2 : 1][2][SQ ? BM : 1];
  __shared__ uint64_t sq_bar[SQ ? 4 : 1];
  constexpr int S = C::STAGES;
  constexpr int NB = C::NBUF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * A_BYTES;
  uint8_t* sSF = sB + S * C::B_BYTES;            // MX: per-stage scale-factor slots
  uint64_t* full = reinterpret_cast<uint64_t*>(sSF + S * C::SF_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + NB;
  uint64_t* drain = tempty + NB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1 + C::SF_WARPS);     // TMA bytes (+ the SF warp's slot)
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    if (SQ)
      for (int i = 0; i < 4; ++i) mbar_init(&sq_bar[i], 2);   // the two warps of a TMEM lane quadrant
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::W_PROD && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == C::W_MMA) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (warp == C::W_PROD && lane == 0) {
    // The first weight tiles of this CTA into L2 while the previous kernel
    // finishes (weights: the MMA's A operand under Swap-AB, else B).
    SegIter si(p);
    Seg g;
    if (si.next(p, g)) {
      const int kend = min(g.kb1, g.kb0 + S);
      for (int kb = g.kb0; kb < kend; ++kb) {
        if (SWAP) tma_prefetch_2d(&tmA, kb * BK, g.ta * BM);
        else tma_prefetch_2d(&tmB, kb * BK, g.tb * BN);
      }
    }
  }
  griddep_wait();
  griddep_launch_dependents();

  auto role_producer = [&]() {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !kTestStallProducer) {
      int it = 0;
      bool ok = true;
      SegIter si(p);
      Seg g;
      while (ok && si.next(p, g)) {
        for (int kb = g.kb0; kb < g.kb1; ++kb, ++it) {
          const int st = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
          tma_load_2d(sA + st * A_BYTES, &tmA, &full[st], kb * BK, g.ta * BM);
          tma_load_2d(sB + st * C::B_BYTES, &tmB, &full[st], kb * BK, g.tb * BN);
        }
      }
      if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        const int first = it - S > 0 ? it - S : 0;
        for (int j = first; j < it; ++j) drain_wait(&full[j % S], (j / S) & 1);
      }
    }
    __syncwarp();
  };
  auto role_mma = [&]() {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = I8 ? idesc_s8_s32(BM, BN) : idesc_e4m3_f32(BM, BN);
      int it = 0, t = 0, pc = 0;
      bool ok = true;
      SegIter si(p);
      Seg g;
      while (ok && si.next(p, g)) {
        const int kb0 = g.kb0, kb1 = g.kb1;
        uint32_t d = tmem_base;
        int buf = 0;
        if (!BW) {
          buf = t % NB;
          if (!mbar_wait(&tempty[buf], ((t / NB) & 1) ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          d = tmem_base + buf * BN;
        }
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int st = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&full[st], ph, abort_flag, p.status)) { ok = false; break; }
          int pb = 0;
          if (BW) {
            pb = pc % NB;
            if (!mbar_wait(&tempty[pb], ((pc / NB) & 1) ^ 1u, abort_flag, p.status)) { ok = false; break; }
            d = tmem_base + pb * BN;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_kmajor_sw128(sA + st * A_BYTES);
          const uint64_t bdesc = smem_desc_kmajor_sw128(sB + st * C::B_BYTES);
          if constexpr (MX) {
            // the stage's scale factors from its shared-memory slot into its
            // TMEM slot, then the four block-scaled MMAs of the stage (a
            // thread's tcgen05 operations run in issue order)
            const uint32_t sf = tmem_base + C::SF_COL0 + st * C::SF_COLS;
            const uint8_t* ssf = sSF + st * C::SF_BYTES;
            tmem_cp_sf_chunk(sf, ssf);
#pragma unroll
            for (int h = 0; h < C::SFB_CHUNKS; ++h) tmem_cp_sf_chunk(sf + 4 + 4 * h, ssf + 512 * (1 + h));
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              const uint32_t acc = (kb > kb0 || k > 0);
              const uint32_t kid = static_cast<uint32_t>(k) << 30;
              mma_mxf8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc_mx_e4m3(BM, BN, k), acc, sf | kid,
                           (sf + 4) | kid);
            }
          } else {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              const uint32_t acc = BW ? (k > 0) : (kb > kb0 || k > 0);
              if constexpr (I8) mma_i8(d, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
              else mma_f8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc, acc);  // +32 bytes of K
            }
          }
          mma_commit(&empty[st]);
          if (BW) {
            mma_commit(&tfull[pb]);
            ++pc;
          }
        }
        if (!ok) break;
        if (!BW) {
          mma_commit(&tfull[buf]);
          ++t;
        }
      }
      // Every MMA issued so far has completed once `drain` flips.
      mma_commit(drain);
      drain_wait(drain, 0);
    }
    __syncwarp();
  };
  auto role_sf = [&]() {
    // ------------------------------------------------------------ scale factors (MX)
    // One warp (on a sub-partition other than the MMA and producer warps').
    // For every stage it writes the E8M0 scale factors into the stage's
    // shared-memory slot -- row l of the SFA chunk: MMA rows l, l+32, l+64,
    // l+96; of SFB chunk h: MMA columns 128 h + l + 32 j; each byte repeated
    // over the stage's four 32-deep K slices -- and arrives on the stage's
    // full barrier; the MMA thread copies the slot into TMEM (tcgen05.cp)
    // right before the stage's MMAs.  (Factors stored into TMEM directly by
    // four warps, one per lane quadrant, were slower: the warp sharing a
    // sub-partition with the MMA thread fell ~3 stages behind.)  A slot is
    // rewritten only after the empty barrier of its stage, so the copies and
    // MMAs that read it have completed.  Rows or columns
    // outside the problem take the scale 1 (byte 127): their operands are
    // zero-filled by TMA.  The scale bytes of a stage are loaded SFD stages
    // ahead (a register ring) so their global latency stays off the path:
    //   no swap: raw[0..3] = A bytes of rows l + 32 j, raw[4..6] = the B
    //            bytes of the (at most three) 128-row weight blocks the
    //            tile's columns fall in;
    //   swap:    raw[0] = the weight block row's byte (the 128 MMA rows are
    //            one block row), raw[1 + 4 h + j] = token column 128 h + l + 32 j.
    constexpr int SFD = 4;
    constexpr int NRAW = SWAP ? 1 + 4 * C::SFB_CHUNKS : 7;
    constexpr uint32_t kOneByte = 127u;
    const int nb_rows = p.N >> 7;                    // weight block rows
    uint32_t raw[SFD][NRAW];
    SegIter sai(p);
    Seg ga;
    bool amore = sai.next(p, ga);
    int akb = amore ? ga.kb0 : 0;
    auto load_ahead = [&](uint32_t* r) {
      if (!amore) {
#pragma unroll
        for (int i = 0; i < NRAW; ++i) r[i] = kOneByte;
        return;
      }
      if (!SWAP) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = ga.ta * BM + lane + 32 * j;
          r[j] = m < p.M ? __ldg(p.sfa + m * p.sfa_sm + akb * p.sfa_skb) : kOneByte;
        }
        const int nb0 = (ga.tb * BN) >> 7;
#pragma unroll
        for (int i = 0; i < 3; ++i)
          r[4 + i] = nb0 + i < nb_rows ? __ldg(p.sfb + (nb0 + i) * p.sfb_snb + akb) : kOneByte;
      } else {
        r[0] = __ldg(p.sfb + ga.ta * p.sfb_snb + akb);
#pragma unroll
        for (int h = 0; h < C::SFB_CHUNKS; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = 128 * h + lane + 32 * j;
            const int m = ga.tb * BN + c;
            r[1 + 4 * h + j] = (c < BN && m < p.M) ? __ldg(p.sfa + m * p.sfa_sm + akb * p.sfa_skb) : kOneByte;
          }
      }
      if (++akb >= ga.kb1) {
        amore = sai.next(p, ga);
        if (amore) akb = ga.kb0;
      }
    };
#pragma unroll
    for (int d = 0; d < SFD; ++d) load_ahead(raw[d]);
    int it = 0;
    bool ok = true;
    SegIter si(p);
    Seg g;
    int tb_cur = -1;
    uint32_t sel[C::SFB_CHUNKS][4];                  // no swap: which raw[4..6] each SFB word takes
    while (ok && si.next(p, g)) {
      if (!SWAP && g.tb != tb_cur) {
        tb_cur = g.tb;
        const int nb0 = (g.tb * BN) >> 7;
#pragma unroll
        for (int h = 0; h < C::SFB_CHUNKS; ++h)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = 128 * h + lane + 32 * j;
            sel[h][j] = c < BN ? static_cast<uint32_t>(((g.tb * BN + c) >> 7) - nb0) : 3u;
          }
      }
      for (int kb = g.kb0; kb < g.kb1; ++kb, ++it) {
        const int st = it % S;
        const uint32_t ph = (it / S) & 1;
        uint32_t cur[NRAW];
#pragma unroll
        for (int i = 0; i < NRAW; ++i) cur[i] = raw[0][i];
#pragma unroll
        for (int d = 0; d + 1 < SFD; ++d)
#pragma unroll
          for (int i = 0; i < NRAW; ++i) raw[d][i] = raw[d + 1][i];
        load_ahead(raw[SFD - 1]);
        uint32_t wa[4], wb[C::SFB_CHUNKS][4];
        if (!SWAP) {
#pragma unroll
          for (int j = 0; j < 4; ++j) wa[j] = cur[j] * 0x01010101u;
#pragma unroll
          for (int h = 0; h < C::SFB_CHUNKS; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t k = sel[h][j];
              wb[h][j] = (k == 0 ? cur[4] : k == 1 ? cur[5] : k == 2 ? cur[6] : kOneByte) * 0x01010101u;
            }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) wa[j] = cur[0] * 0x01010101u;
#pragma unroll
          for (int h = 0; h < C::SFB_CHUNKS; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) wb[h][j] = cur[1 + 4 * h + j] * 0x01010101u;
        }
        int w_ok = 1;
        if (lane == 0) w_ok = mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status);
        if (!__shfl_sync(0xFFFFFFFFu, w_ok, 0)) { ok = false; break; }
        // row `lane` of each 512-byte chunk: the factors of MMA rows (or
        // columns) lane, lane + 32, lane + 64, lane + 96
        uint32_t* sf = reinterpret_cast<uint32_t*>(sSF + st * C::SF_BYTES);
        *reinterpret_cast<uint4*>(sf + lane * 4) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
#pragma unroll
        for (int h = 0; h < C::SFB_CHUNKS; ++h)
          *reinterpret_cast<uint4*>(sf + 128 * (1 + h) + lane * 4) =
              make_uint4(wb[h][0], wb[h][1], wb[h][2], wb[h][3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[st]);
      }
    }
    __syncwarp();
  };
  auto role_epilogue = [&]() {
    // ------------------------------------------------------------ epilogue
    const int e = warp - C::EPI_BASE;
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int cg = e >> 2;                     // column slice
    const int row = quad * 32 + lane;          // MMA-A row within the tile
    const int col0 = cg * C::CPT;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int t = 0, pc = 0, sq_t = 0;
    bool ok = true;

    SegIter si(p);
    Seg g;
    while (ok && si.next(p, g)) {
      const int ta = g.ta, tb = g.tb, kb0 = g.kb0, kb1 = g.kb1;
      const int a_idx = ta * BM + row;                         // m (no swap) or n (swap)
      const int b_base = tb * BN;                              // first column's n or m
      const bool a_valid = a_idx < (SWAP ? p.N : p.M);
      const int tile_id = tb * p.tiles_a + ta;
      float* ws_tile = p.ws + (static_cast<int64_t>(tile_id) * p.max_contrib) * (BN * BM);

      // Store one chunk of CHUNK final values v[] for columns col..col+CHUNK-1.
      auto emit = [&](int col, const float* v) {
        if (!a_valid) return;
        if (!SWAP) {
          const int m = a_idx;
          uint16_t* yr = p.y + static_cast<int64_t>(m) * p.ldy;
#pragma unroll
          for (int g = 0; g < C::CHUNK; g += 8) {
            const int n = b_base + col + g;
            if (n < p.N) {
              uint4 o;
              o.x = pack_bf16x2(v[g + 0], v[g + 1]);
              o.y = pack_bf16x2(v[g + 2], v[g + 3]);
              o.z = pack_bf16x2(v[g + 4], v[g + 5]);
              o.w = pack_bf16x2(v[g + 6], v[g + 7]);
              *reinterpret_cast<uint4*>(yr + n) = o;
            }
          }
        } else {
          const int n = a_idx;
#pragma unroll
          for (int i = 0; i < C::CHUNK; ++i) {
            const int m = b_base + col + i;
            if (m < p.M)
              p.y[static_cast<int64_t>(m) * p.ldy + n] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
          }
        }
      };
      // Partial layout inside a slot.  VEC: [col/4][row][4] fp32, each lane
      // moving 16 bytes, a warp's access 512 contiguous bytes.  Otherwise
      // (the 16-warp variant, whose register budget is tight): [col][row],
      // 4 bytes a lane, 128 contiguous bytes a warp.
      constexpr bool VEC = C::EPI_WARPS < 16;
      auto stash = [&](int col, const float* v) {    // fp32 partial of this piece
        float* w = ws_tile + static_cast<int64_t>(g.slot) * (BN * BM);
        if (VEC) {
#pragma unroll
          for (int i = 0; i < C::CHUNK; i += 4)
            __stcg(reinterpret_cast<float4*>(w) + ((col + i) >> 2) * BM + row,
                   make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < C::CHUNK; ++i) __stcg(w + (col + i) * BM + row, v[i]);
        }
      };
      auto finish_split = [&]() {                    // last arrival sums the partials in order
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(&p.counters[tile_id * C::EPI_WARPS + e], 1);
        old = __shfl_sync(0xFFFFFFFFu, old, 0);
        if (old != g.ncontrib - 1) return;
        if (lane == 0) p.counters[tile_id * C::EPI_WARPS + e] = 0;
        __threadfence();
        // Slots are added in slot order (VEC: two slots' loads in flight at once).
        constexpr int Q = C::CHUNK / 4;
        constexpr int64_t SLOT = BN * BM;
        for (int c = col0; c < col0 + C::CPT; c += C::CHUNK) {
          float v[C::CHUNK];
#pragma unroll
          for (int i = 0; i < C::CHUNK; ++i) v[i] = 0.0f;
          if (VEC) {
            const float4* wc = reinterpret_cast<const float4*>(ws_tile) + (c >> 2) * BM + row;
            int ss = 0;
            for (; ss + 1 < g.ncontrib; ss += 2) {
              float4 x0[Q], x1[Q];
#pragma unroll
              for (int i = 0; i < Q; ++i) x0[i] = __ldcg(wc + ss * (SLOT / 4) + i * BM);
#pragma unroll
              for (int i = 0; i < Q; ++i) x1[i] = __ldcg(wc + (ss + 1) * (SLOT / 4) + i * BM);
#pragma unroll
              for (int i = 0; i < Q; ++i) {
                v[4 * i + 0] += x0[i].x; v[4 * i + 1] += x0[i].y; v[4 * i + 2] += x0[i].z; v[4 * i + 3] += x0[i].w;
              }
#pragma unroll
              for (int i = 0; i < Q; ++i) {
                v[4 * i + 0] += x1[i].x; v[4 * i + 1] += x1[i].y; v[4 * i + 2] += x1[i].z; v[4 * i + 3] += x1[i].w;
              }
            }
            if (ss < g.ncontrib) {
#pragma unroll
              for (int i = 0; i < Q; ++i) {
                const float4 x = __ldcg(wc + ss * (SLOT / 4) + i * BM);
                v[4 * i + 0] += x.x; v[4 * i + 1] += x.y; v[4 * i + 2] += x.z; v[4 * i + 3] += x.w;
              }
            }
          } else {
            for (int ss = 0; ss < g.ncontrib; ++ss) {
              const float* w = ws_tile + ss * SLOT;
#pragma unroll
              for (int i = 0; i < C::CHUNK; ++i) v[i] += __ldcg(w + (c + i) * BM + row);
            }
          }
          emit(c, v);
        }
      };

      if constexpr (!BW) {
        // -------- per-token / per-channel scales: one accumulator per tile
        // Column scales: lane l of the warp loads the scale of column c + l of
        // every chunk (one load per 32 columns, issued before the wait), and the
        // products broadcast it with a shuffle.
        constexpr int NCH = C::CPT / C::CHUNK;
        const int buf = t % NB;
        float srow = 1.0f;
        float colsc[NCH];
        if constexpr (!MX) {
          if (!SWAP) srow = a_valid ? __ldg(p.sa + a_idx * p.sa_sm) : 0.0f;
          else srow = a_valid ? __ldg(p.sb + a_idx * p.sb_sn) : 0.0f;
#pragma unroll
          for (int j = 0; j < NCH; ++j) {
            const int b_idx = b_base + col0 + j * C::CHUNK + lane;
            if (!SWAP) colsc[j] = (lane < C::CHUNK && b_idx < p.N) ? __ldg(p.sb + b_idx * p.sb_sn) : 0.0f;
            else colsc[j] = (lane < C::CHUNK && b_idx < p.M) ? __ldg(p.sa + b_idx * p.sa_sm) : 0.0f;
          }
        }
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[buf], (t / NB) & 1, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          const int c = col0 + j * C::CHUNK;
          uint32_t r[C::CHUNK];
          tmem_ld_waited<C::CHUNK>(tmem_base + lane_addr + buf * BN + c, r);
          float v[C::CHUNK];
#pragma unroll
          for (int i = 0; i < C::CHUNK; ++i) {
            if constexpr (MX) v[i] = __uint_as_float(r[i]);
            else if constexpr (I8)   // exact s32 sum -> fp32 (one rounding beyond 2^24)
              v[i] = __int2float_rn(static_cast<int>(r[i])) * (srow * __shfl_sync(0xFFFFFFFFu, colsc[j], i));
            else v[i] = __uint_as_float(r[i]) * (srow * __shfl_sync(0xFFFFFFFFu, colsc[j], i));
          }
          if (g.ncontrib == 1) emit(c, v);
          else stash(c, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        ++t;
        if (g.ncontrib > 1) finish_split();
      } else {
        // -------- blockwise scales: promote each K-block partial into registers.
        // The raw scales of the next SD K blocks are kept in flight in a
        // register ring (stage 0 = the block being promoted), so the
        // global-load latency of a block's scales overlaps the promotion of
        // the blocks before it; the product sa * sb is formed only when the
        // block is consumed (forming it at load time would wait for the load
        // right there).  Swap-AB: the scale varies per column (token); lane l
        // holds that of column c + l of every chunk.
        constexpr int NCH = C::CPT / C::CHUNK;
        constexpr int SD = 3;
        uint64_t acc[C::CPT / 2];                      // fp32 pairs, columns 2i, 2i+1
#pragma unroll
        for (int i = 0; i < C::CPT / 2; ++i) acc[i] = 0ull;
        // Scale offsets (elements; every scale array is far below 2^31 of
        // them) advance one K block per load.  A row or column outside the
        // problem reads the scales of row/column 0 instead: its output is never
        // written.  Weight block row: the whole tile (Swap-AB) or this warp's
        // 128-column slice (a slice never straddles a block row).
        // (SQ: the slice spans the tile's gate block row 2 tb and up block row 2 tb + 1)
        const int nb = SWAP ? ta : (SQ ? 2 * tb : (tb * BN + col0) / 128);
        const bool slice_valid = SWAP || (tb * BN + col0) < p.N;
        int sb_o = static_cast<int>((slice_valid ? nb : 0) * p.sb_snb + kb0 * p.sb_skb);
        int sb_o2 = SQ ? static_cast<int>((nb + 1) * p.sb_snb + kb0 * p.sb_skb) : 0;
        int sa_o[SWAP ? NCH : 1];
        if (!SWAP) {
          sa_o[0] = static_cast<int>((a_valid ? a_idx : 0) * p.sa_sm + kb0 * p.sa_skb);
        } else {
#pragma unroll
          for (int j = 0; j < NCH; ++j) {
            const int m = b_base + col0 + j * C::CHUNK + lane;
            sa_o[j] = static_cast<int>((m < p.M ? m : 0) * p.sa_sm + kb0 * p.sa_skb);
          }
        }
        constexpr int NSC = SWAP ? NCH : (SQ ? 2 : 1);  // scales per K block per thread
        constexpr int NA = SWAP ? NCH : 1;             // activation scales per K block
        constexpr int NW = SQ ? 2 : 1;                 // weight scales per K block (SQ: gate, up)
        float ra[SD][NA], rw[SD][NW];
        int kl = kb0;                                  // next K block to load scales of
        auto load_scales = [&](float* a_out, float* w_out) {
          const bool in = kl < kb1;
          w_out[0] = in ? __ldg(p.sb + sb_o) : 0.0f;
          if constexpr (SQ) {
            w_out[NW - 1] = in ? __ldg(p.sb + sb_o2) : 0.0f;
            sb_o2 += static_cast<int>(p.sb_skb);
          }
#pragma unroll
          for (int j = 0; j < NA; ++j) {
            a_out[j] = in ? __ldg(p.sa + sa_o[j]) : 0.0f;
            sa_o[j] += static_cast<int>(p.sa_skb);
          }
          sb_o += static_cast<int>(p.sb_skb);
          ++kl;
        };
#pragma unroll
        for (int q = 0; q < SD; ++q) load_scales(ra[q], rw[q]);
        int pb = pc % NB;
        uint32_t ph = (pc / NB) & 1;
        for (int kb = kb0; kb < kb1; ++kb) {
          float sc0[NSC];                              // sa * sb (SQ: gate, up)
#pragma unroll
          for (int j = 0; j < NSC; ++j) sc0[j] = ra[0][SWAP ? j : 0] * rw[0][SQ ? j : 0];
#pragma unroll
          for (int q = 0; q + 1 < SD; ++q) {
#pragma unroll
            for (int j = 0; j < NA; ++j) ra[q][j] = ra[q + 1][j];
#pragma unroll
            for (int j = 0; j < NW; ++j) rw[q][j] = rw[q + 1][j];
          }
          load_scales(ra[SD - 1], rw[SD - 1]);
          const uint64_t srow2 = pair_f32(sc0[0], sc0[0]);
          const uint64_t srow2u = pair_f32(sc0[NSC - 1], sc0[NSC - 1]);   // SQ: up half
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[pb], ph, abort_flag, p.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Chunk j + 1 is loaded while chunk j is scaled into the
          // accumulators; the buffer is handed back to the MMA as soon as the
          // last chunk has landed, before its FMAs.
          // (SQ: chunk j < NCH/2 is gate column 64 cg + 8 j of the tile,
          // chunk j >= NCH/2 the matching up column 128 + 64 cg + 8 (j - NCH/2))
          const uint32_t tbuf = tmem_base + lane_addr + pb * BN + (SQ ? 0 : col0);
          auto ccol = [&](int j) {
            return SQ ? (j < NCH / 2 ? 64 * cg + j * C::CHUNK : 128 + 64 * cg + (j - NCH / 2) * C::CHUNK)
                      : j * C::CHUNK;
          };
          uint32_t r[2][C::CHUNK];
          tmem_ld_async<C::CHUNK>(tbuf + ccol(0), r[0]);
#pragma unroll
          for (int j = 0; j < NCH; ++j) {
            uint32_t* rc = r[j & 1];
            tmem_wait_regs<C::CHUNK>(rc);
            if (j + 1 < NCH) {
              tmem_ld_async<C::CHUNK>(tbuf + ccol(j + 1), r[(j + 1) & 1]);
            } else {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[pb]);
            }
#pragma unroll
            for (int i = 0; i < C::CHUNK; i += 2) {
              const uint64_t sc = SWAP ? pair_f32(__shfl_sync(0xFFFFFFFFu, sc0[SWAP ? j : 0], i),
                                                  __shfl_sync(0xFFFFFFFFu, sc0[SWAP ? j : 0], i + 1))
                                       : ((SQ && j >= NCH / 2) ? srow2u : srow2);
              ffma2_acc(acc[(j * C::CHUNK + i) / 2], rc[i], rc[i + 1], sc);
            }
          }
          if (++pb == NB) {
            pb = 0;
            ph ^= 1u;
          }
          ++pc;
        }
        if (!ok) break;
        if constexpr (SQ) {
          // gate values in acc[0, 32), up values in acc[32, 64) (pairs);
          // h = bf16 of each, as the GEMM emits y; y = bf16(silu(h_gate) h_up)
          // Each pair's value is the bf16 rounding of the low end of its
          // bracket.  A pair whose bracket straddles a rounding midpoint
          // ("open") is within one bf16 step of its exact value; in the exact
          // mode, and for tiny values or gates below -85 always, its chunk is
          // recomputed exactly right away.  In the fast mode an open chunk is
          // recomputed only if it can decide the group amax (within
          // kCandSteps of this slice's amax: the slice's exact amax is then
          // exact, and the partner slice's likewise), so scales stay exact
          // and codes differ from the exact ones only where an open y does.
          // (Open pairs are rare, ~1e-3 of the values, but an exact
          // recomputation in a warp stalls the whole tile's epilogue.)
          uint4 gv[8], uv[8];                          // h = bf16 of the sums, 8 chunks
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t gw[4], uw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float a0, a1, b0, b1;
              unpair_f32(acc[4 * c + k], a0, a1);
              unpair_f32(acc[32 + 4 * c + k], b0, b1);
              gw[k] = pack_bf16x2(a0, a1);
              uw[k] = pack_bf16x2(b0, b1);
            }
            gv[c] = make_uint4(gw[0], gw[1], gw[2], gw[3]);
            uv[c] = make_uint4(uw[0], uw[1], uw[2], uw[3]);
          }
          uint4 yv[8];
          uint32_t m2 = 0, open = 0;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t gw[4] = {gv[c].x, gv[c].y, gv[c].z, gv[c].w};
            const uint32_t uw[4] = {uv[c].x, uv[c].y, uv[c].z, uv[c].w};
            uint32_t d = 0;
            bool bad = false;
            uint4 y;
            y.x = silu_pair(gw[0], uw[0], d, bad);
            y.y = silu_pair(gw[1], uw[1], d, bad);
            y.z = silu_pair(gw[2], uw[2], d, bad);
            y.w = silu_pair(gw[3], uw[3], d, bad);
            if (bad || (d != 0 && p.sq_exact))
              y = silu_chunk_fix(gv[c], uv[c], y);
            else
              open |= static_cast<uint32_t>(d != 0) << c;
            yv[c] = y;
            m2 = chunk_absmax2(y, m2);
          }
          if (open) {
            const float thr = bf16_steps_below(absmax2_to_f32(m2), kCandSteps);
            m2 = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              if (((open >> c) & 1u) && absmax2_to_f32(chunk_absmax2(yv[c], 0u)) >= thr)
                yv[c] = silu_chunk_fix(gv[c], uv[c], yv[c]);
              m2 = chunk_absmax2(yv[c], m2);
            }
          }
          // group amax over the two column slices of the row: write this
          // slice's partial, one arrival per warp, bounded wait for the
          // partner warp (same lane quadrant), read its partial.  The slot of
          // tile t is written again at tile t + 2, after both warps have arrived for
          // tile t + 1, so the partner has read it.
          float am = absmax2_to_f32(m2);
          const int par = sq_t & 1;
          sq_red[par][cg][row] = am;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sq_bar[quad]);
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sq_bar[quad], static_cast<uint32_t>(par), abort_flag, p.status))) {
            ok = false;
            break;
          }
          am = fmaxf(am, sq_red[par][cg ^ 1][row]);
          ++sq_t;
          const QScale qs = make_qscale(am, p.sq_ue8m0);
          if (a_valid) {
            uint8_t* qr = p.sq_q + static_cast<int64_t>(a_idx) * p.sq_ldq + tb * 128 + 64 * cg;
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint2*>(qr + 8 * c) = quant_chunk(yv[c], qs);
            if (cg == 0) {
              const int64_t si = static_cast<int64_t>(a_idx) * p.sq_s_sm + static_cast<int64_t>(tb) * p.sq_s_sg;
              if (p.sq_ue8m0 == 2) reinterpret_cast<uint8_t*>(p.sq_s)[si] = static_cast<uint8_t>(__float_as_uint(qs.s) >> 23);
              else p.sq_s[si] = qs.s;
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < C::CPT; c += C::CHUNK) {
            float v[C::CHUNK];
#pragma unroll
            for (int i = 0; i < C::CHUNK; i += 2) unpair_f32(acc[(c + i) / 2], v[i], v[i + 1]);
            if (g.ncontrib == 1) emit(col0 + c, v);
            else stash(col0 + c, v);
          }
          if (g.ncontrib > 1) finish_split();
        }
      }
    }
  };
  if constexpr (C::REGSPLIT) {
    // the third warpgroup (producer, MMA, two idle warps) gives up registers,
    // the two epilogue warpgroups take them; each role body sits inside its
    // warpgroup's branch so its code is allocated under the new limit
    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegLow));
      if (warp == C::W_PROD) role_producer();
      else if (warp == C::W_MMA) role_mma();
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegHigh));
      role_epilogue();
    }
  } else {
    if (warp == C::W_PROD) role_producer();
    else if (warp == C::W_MMA) role_mma();
    else if (MX && warp >= 2 + C::EPI_WARPS) role_sf();   // (MX kernels have no register split)
    else if (warp >= C::EPI_BASE && warp < C::EPI_BASE + C::EPI_WARPS) role_epilogue();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::W_MMA) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ------------------------------------------------------------------ CTA pairs
// Pair kernel: a cluster of two CTAs (on two SMs) computes one 256 x BN tile
// with tcgen05 .cta_group::2 MMAs.  CTA rank r loads rows [128 r, 128 r + 128)
// of the A tile and rows [BN/2 r, BN/2 r + BN/2) of the B tile into its own
// shared memory, and its TMEM receives rows [128 r, 128 r + 128) of the
// accumulator; the even CTA issues the MMAs (M = 256, N = BN) and every
// completion is multicast to both CTAs' mbarriers.  Each SM thus stages half
// a B tile per K block: a 128-column tile costs it the shared-memory traffic
// of a 256-column single-CTA tile while TMEM keeps room for four 128-column
// accumulator buffers -- for the blockwise scheme three K blocks of slack
// between the MMA and the promotion epilogue instead of one.
// Both CTAs' TMA loads count their bytes on the even CTA's full barrier (no
// multicast loads); the epilogue warps of both CTAs release an accumulator
// buffer on the even CTA's tempty barrier.  A cluster barrier precedes any
// cross-CTA use of the barriers and the TMEM release.
template <int BN, bool BW>
struct Cfg2 {
  static constexpr int HB = BN / 2;                        // B rows per CTA
  static constexpr int B_BYTES = HB * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // per CTA
  static constexpr int STAGES_RAW = kSmemBudget / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int NBUF = (512 / BN) > 4 ? 4 : (512 / BN);
  static constexpr int EPI_WARPS = BW ? (BN >= 256 ? 16 : 8) : 4;
  static constexpr int COL_GROUPS = EPI_WARPS / 4;
  static constexpr int CPT = BN / COL_GROUPS;
  static constexpr int CHUNK = 32;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * NBUF + 1) + 16;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static_assert(NBUF * BN <= 512, "accumulators exceed TMEM");
  static_assert(CPT % CHUNK == 0, "chunking");
  static_assert(B_BYTES % 1024 == 0, "B tiles must stay 1024-byte aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int BN, bool BW, bool I8 = false>
__global__ void __launch_bounds__(Cfg2<BN, BW>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmArgs p) {
  using C = Cfg2<BN, BW>;
  constexpr int S = C::STAGES;
  constexpr int NB = C::NBUF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * C::B_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + NB;
  uint64_t* drain = tempty + NB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < NB; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int pair = static_cast<int>(blockIdx.x >> 1);
  if (warp == 0 && lane == 0 && pair < p.units) {
    // this CTA's half of the first weight tiles into L2 (see gemm_kernel)
    const int tb = pair / p.tiles_a;
    const int kend = min(p.kblocks, S);
    for (int kb = 0; kb < kend; ++kb)
      tma_prefetch_2d(&tmB, kb * BK, tb * BN + static_cast<int>(rank) * C::HB);
  }
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = pair; ok && u < p.units; u += npairs) {
        const int ta = u % p.tiles_a, tb = u / p.tiles_a;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int st = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[st], 2 * C::STAGE_BYTES);
          const uint32_t fb = mapa_shared(smem_u32(&full[st]), 0);
          tma_load_2d_pair(sA + st * A_BYTES, &tmA, fb, kb * BK, ta * (2 * BM) + static_cast<int>(rank) * BM);
          tma_load_2d_pair(sB + st * C::B_BYTES, &tmB, fb, kb * BK, tb * BN + static_cast<int>(rank) * C::HB);
        }
      }
      if (leader) {
        // Let the copies of both CTAs land (they count on these barriers)
        // before the pair can leave (immediate when everything was consumed).
        const int first = it - S > 0 ? it - S : 0;
        for (int j = first; j < it; ++j) drain_wait(&full[j % S], (j / S) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = I8 ? idesc_s8_s32(2 * BM, BN) : idesc_e4m3_f32(2 * BM, BN);
      int it = 0, t = 0, pc = 0;
      bool ok = true;
      for (int u = pair; ok && u < p.units; u += npairs) {
        uint32_t d = tmem_base;
        int buf = 0;
        if (!BW) {
          buf = t % NB;
          if (!mbar_wait(&tempty[buf], ((t / NB) & 1) ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          d = tmem_base + buf * BN;
        }
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int st = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(&full[st], ph, abort_flag, p.status)) { ok = false; break; }
          int pb = 0;
          if (BW) {
            pb = pc % NB;
            if (!mbar_wait(&tempty[pb], ((pc / NB) & 1) ^ 1u, abort_flag, p.status)) { ok = false; break; }
            d = tmem_base + pb * BN;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_kmajor_sw128(sA + st * A_BYTES);
          const uint64_t bdesc = smem_desc_kmajor_sw128(sB + st * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint32_t acc = BW ? (k > 0) : (kb > 0 || k > 0);
            if constexpr (I8) mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
            else mma_f8f6f4_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
          }
          mma_commit_pair(&empty[st], 0x3);
          if (BW) {
            mma_commit_pair(&tfull[pb], 0x3);
            ++pc;
          }
        }
        if (!ok) break;
        if (!BW) {
          mma_commit_pair(&tfull[buf], 0x3);
          ++t;
        }
      }
      // Every MMA issued so far, which reads both CTAs' shared memory, has
      // completed once `drain` flips in both CTAs.
      mma_commit_pair(drain, 0x3);
    }
    if (lane == 0) drain_wait(drain, 0);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int e = warp - 2;
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int cg = e >> 2;                     // column slice
    const int row = quad * 32 + lane;          // accumulator row within this CTA's half
    const int col0 = cg * C::CPT;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    constexpr int NCH = C::CPT / C::CHUNK;
    int t = 0, pc = 0;
    bool ok = true;
    for (int u = pair; ok && u < p.units; u += npairs) {
      const int ta = u % p.tiles_a, tb = u / p.tiles_a;
      const int m = ta * (2 * BM) + static_cast<int>(rank) * BM + row;
      const bool m_valid = m < p.M;
      uint16_t* yr = p.y + static_cast<int64_t>(m_valid ? m : 0) * p.ldy;
      auto emit = [&](int col, const float* v) {
        if (!m_valid) return;
#pragma unroll
        for (int g8 = 0; g8 < C::CHUNK; g8 += 8) {
          const int n = tb * BN + col + g8;
          if (n < p.N) {
            uint4 o;
            o.x = pack_bf16x2(v[g8 + 0], v[g8 + 1]);
            o.y = pack_bf16x2(v[g8 + 2], v[g8 + 3]);
            o.z = pack_bf16x2(v[g8 + 4], v[g8 + 5]);
            o.w = pack_bf16x2(v[g8 + 6], v[g8 + 7]);
            *reinterpret_cast<uint4*>(yr + n) = o;
          }
        }
      };
      if (!BW) {
        // -------- per-token / per-channel scales: one accumulator per tile
        const int buf = t % NB;
        const float srow = m_valid ? __ldg(p.sa + m * p.sa_sm) : 0.0f;
        float colsc[NCH];
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          const int n = tb * BN + col0 + j * C::CHUNK + lane;
          colsc[j] = n < p.N ? __ldg(p.sb + n * p.sb_sn) : 0.0f;
        }
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[buf], (t / NB) & 1, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          uint32_t r[C::CHUNK];
          tmem_ld_waited<C::CHUNK>(tmem_base + lane_addr + buf * BN + col0 + j * C::CHUNK, r);
          float v[C::CHUNK];
#pragma unroll
          for (int i = 0; i < C::CHUNK; ++i) {
            const float a = I8 ? __int2float_rn(static_cast<int>(r[i])) : __uint_as_float(r[i]);
            v[i] = a * (srow * __shfl_sync(0xFFFFFFFFu, colsc[j], i));
          }
          emit(col0 + j * C::CHUNK, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * buf);
        ++t;
      } else {
        // -------- blockwise scales: promote each K-block partial into registers
        uint64_t acc[C::CPT / 2];
#pragma unroll
        for (int i = 0; i < C::CPT / 2; ++i) acc[i] = 0ull;
        const int nb = (tb * BN + col0) / 128;
        const bool slice_valid = (tb * BN + col0) < p.N;
        // raw scales of the next SD K blocks in flight; sa * sb formed on use
        constexpr int SD = 4;
        float ra[SD], rw[SD];
        auto load_scale = [&](int kb, float& a, float& w) {
          const bool in = kb < p.kblocks && slice_valid && m_valid;
          a = in ? __ldg(p.sa + m * p.sa_sm + kb * p.sa_skb) : 0.0f;
          w = in ? __ldg(p.sb + nb * p.sb_snb + kb * p.sb_skb) : 0.0f;
        };
#pragma unroll
        for (int q = 0; q < SD; ++q) load_scale(q, ra[q], rw[q]);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          const int pb = pc % NB;
          const float s0 = ra[0] * rw[0];
          const uint64_t srow2 = pair_f32(s0, s0);
#pragma unroll
          for (int q = 0; q + 1 < SD; ++q) {
            ra[q] = ra[q + 1];
            rw[q] = rw[q + 1];
          }
          load_scale(kb + SD, ra[SD - 1], rw[SD - 1]);
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&tfull[pb], (pc / NB) & 1, abort_flag, p.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // All of this warp's columns are read with one wait, the buffer is
          // handed back, then the partial is scaled into the accumulators.
          uint32_t r[NCH][C::CHUNK];
#pragma unroll
          for (int j = 0; j < NCH; ++j)
            tmem_ld_32x32b_x32_raw(tmem_base + lane_addr + pb * BN + col0 + j * C::CHUNK, r[j]);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * pb);
#pragma unroll
          for (int j = 0; j < NCH; ++j)
#pragma unroll
            for (int i = 0; i < C::CHUNK; i += 2)
              ffma2_acc(acc[(j * C::CHUNK + i) / 2], r[j][i], r[j][i + 1], srow2);
          ++pc;
        }
        if (!ok) break;
#pragma unroll
        for (int c = 0; c < C::CPT; c += C::CHUNK) {
          float v[C::CHUNK];
#pragma unroll
          for (int i = 0; i < C::CHUNK; i += 2) unpair_f32(acc[(c + i) / 2], v[i], v[i + 1]);
          emit(col0 + c, v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

// ------------------------------------------------------------------ decode (M <= 8)
// At M <= 8 tokens a linear layer is bound by reading its weights once from
// HBM (N K bytes; 52 MB for the Qwen3-32B qkv projection) and does only 2 M
// flops per weight byte, so this kernel streams the weights with 16-byte
// loads straight into the registers of the warp-level MMA
// (mma.sync.m16n8k32, e4m3 x e4m3 -> f32: the weight rows in its 16-row slot,
// the tokens in its 8 columns, absent tokens as zeros).  There is no TMEM
// allocation, no tensor-map setup and no split-K round trip through global
// memory: a CTA owns 16 weight rows, its kDecodeWarps warps split K, and their
// partial sums meet once in shared memory.
// K order inside a 64-deep chunk: lane (g, t) = (lane / 4, lane % 4) loads the
// 16 contiguous bytes [16 t, 16 t + 16) of weight rows g and g + 8 and of token
// g; bytes 0-7 feed the chunk's first MMA and 8-15 its second.  The MMA's own
// k order inside an instruction differs, but every product a[m][k] b[n][k] of
// the chunk is formed exactly once, and a chunk never straddles a 128-deep
// block, so the blockwise scales apply to the right sums.
// Scales as in the tcgen05 kernels: blockwise, each K block's fp32 partial
// times sa[m, kb] sb[n / 128, kb] into the fp32 total; per token, the total
// times sa[m] sb[n] at the end.
constexpr int kDecodeWarps = 8;
constexpr int kDecodeRows = 16;
constexpr int kDecodeMaxM = 8;

__device__ __forceinline__ void mma_e4m3_m16n8k32(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                                  uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_weight(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <bool BW>
__global__ void __launch_bounds__(32 * kDecodeWarps) decode_kernel(const uint8_t* __restrict__ a,
                                                                   const uint8_t* __restrict__ b,
                                                                   const GemmArgs p) {
  __shared__ float red[kDecodeWarps][kDecodeRows][kDecodeMaxM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = static_cast<int>(blockIdx.x) * kDecodeRows;
  const int kblocks = p.K / BK;
  const int kb0 = (kblocks * warp) / kDecodeWarps, kb1 = (kblocks * (warp + 1)) / kDecodeWarps;
  const uint8_t* w0 = b + static_cast<int64_t>(n0 + g) * p.K + 16 * t;
  const uint8_t* w1 = w0 + 8LL * p.K;
  const bool tok = g < p.M;
  const uint8_t* ar = a + static_cast<int64_t>(tok ? g : 0) * p.K + 16 * t;
  griddep_wait();                       // activations and scales may come from the previous kernel
  griddep_launch_dependents();
  // one K block = two 64-deep chunks
  auto load = [&](int kb, uint4* wa, uint4* wb, uint4* av) {
    const int64_t k0 = static_cast<int64_t>(kb) * BK;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      wa[c] = ld_weight(w0 + k0 + 64 * c);
      wb[c] = ld_weight(w1 + k0 + 64 * c);
      av[c] = tok ? __ldg(reinterpret_cast<const uint4*>(ar + k0 + 64 * c)) : make_uint4(0, 0, 0, 0);
    }
  };
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  auto compute = [&](int kb, const uint4* wa, const uint4* wb, const uint4* av) {
    float cc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float* d = BW ? cc : acc;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      mma_e4m3_m16n8k32(d, wa[c].x, wb[c].x, wa[c].y, wb[c].y, av[c].x, av[c].y);
      mma_e4m3_m16n8k32(d, wa[c].z, wb[c].z, wa[c].w, wb[c].w, av[c].z, av[c].w);
    }
    if constexpr (BW) {
      // C fragment: cc[0], cc[1] = rows g, tokens 2t, 2t+1; cc[2], cc[3] = row g + 8
      const float sbk = __ldg(p.sb + (n0 / 128) * p.sb_snb + kb * p.sb_skb);
      const float s0 = 2 * t < p.M ? __ldg(p.sa + (2 * t) * p.sa_sm + kb * p.sa_skb) * sbk : 0.0f;
      const float s1 = 2 * t + 1 < p.M ? __ldg(p.sa + (2 * t + 1) * p.sa_sm + kb * p.sa_skb) * sbk : 0.0f;
      acc[0] = fmaf(cc[0], s0, acc[0]);
      acc[1] = fmaf(cc[1], s1, acc[1]);
      acc[2] = fmaf(cc[2], s0, acc[2]);
      acc[3] = fmaf(cc[3], s1, acc[3]);
    }
  };
  // a ring of three K blocks in registers: block kb + 3's loads are issued as
  // soon as block kb's MMAs have read their operands
  uint4 a0[2], b0[2], v0[2], a1[2], b1[2], v1[2], a2[2], b2[2], v2[2];
  if (kb0 < kb1) load(kb0, a0, b0, v0);
  if (kb0 + 1 < kb1) load(kb0 + 1, a1, b1, v1);
  if (kb0 + 2 < kb1) load(kb0 + 2, a2, b2, v2);
  for (int kb = kb0; kb < kb1; kb += 3) {
    compute(kb, a0, b0, v0);
    if (kb + 3 < kb1) load(kb + 3, a0, b0, v0);
    if (kb + 1 < kb1) compute(kb + 1, a1, b1, v1);
    if (kb + 4 < kb1) load(kb + 4, a1, b1, v1);
    if (kb + 2 < kb1) compute(kb + 2, a2, b2, v2);
    if (kb + 5 < kb1) load(kb + 5, a2, b2, v2);
  }
  red[warp][g][2 * t] = acc[0];
  red[warp][g][2 * t + 1] = acc[1];
  red[warp][g + 8][2 * t] = acc[2];
  red[warp][g + 8][2 * t + 1] = acc[3];
  __syncthreads();
  // the warps' partials in warp order; one thread per (row, token)
  if (threadIdx.x < kDecodeRows * kDecodeMaxM) {
    const int r = threadIdx.x / kDecodeMaxM, m = threadIdx.x % kDecodeMaxM;
    if (m < p.M) {
      float v = red[0][r][m];
#pragma unroll
      for (int w = 1; w < kDecodeWarps; ++w) v += red[w][r][m];
      if constexpr (!BW) v *= __ldg(p.sa + m * p.sa_sm) * __ldg(p.sb + (n0 + r) * p.sb_sn);
      p.y[static_cast<int64_t>(m) * p.ldy + n0 + r] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

struct MapKey {
  const void* ptr;
  int64_t rows, k;
  int box_rows, dev;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && rows == o.rows && k == o.k && box_rows == o.box_rows && dev == o.dev;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = reinterpret_cast<uintptr_t>(k.ptr);
    h ^= static_cast<size_t>(k.rows) * 0x9E3779B97F4A7C15ull;
    h ^= static_cast<size_t>(k.k) * 0xC2B2AE3D27D4EB4Full;
    h ^= static_cast<size_t>(k.box_rows) * 0x165667B19E3779F9ull + static_cast<size_t>(k.dev);
    return h;
  }
};

// Tensor map of an e4m3 [rows, k] row-major matrix, box = box_rows x 128
// bytes, 128-byte swizzle, zero fill outside the matrix.  Cached per
// (pointer, shape, box, device).
bool tensor_map(const void* ptr, int64_t rows, int64_t k, int box_rows, CUtensorMap* out) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const MapKey key{ptr, rows, k, box_rows, dev};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *out = it->second;
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMap m;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(k)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), gdim,
                        gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() > 4096) cache.clear();
  cache.emplace(key, m);
  *out = m;
  return true;
}

template <int BN, bool SWAP, bool BW, bool MX = false, bool I8 = false, bool SQ = false>
fp8q_status launch_gemm(const void* a_op, const void* b_op, const GemmArgs& p,
                        cudaStream_t stream) {
  using C = Cfg<BN, SWAP, BW, MX, I8>;
  CUtensorMap ma, mb;
  if (!tensor_map(a_op, p.rows_a, p.K, BM, &ma) || !tensor_map(b_op, p.rows_b, p.K, BN, &mb))
    return FP8Q_ERR_CUDA;
  static std::atomic<int> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(gemm_kernel<BN, SWAP, BW, MX, I8, SQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr_done[dev].store(1, std::memory_order_relaxed);
  }
  int grid;
  if (p.streamk) grid = (p.total_iters + p.seg_len - 1) / p.seg_len;
  else grid = p.units < num_sms() ? p.units : num_sms();
  return launch_kernel(gemm_kernel<BN, SWAP, BW, MX, I8, SQ>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES,
                       stream, 1, ma, mb, p);
}

// Clusters of two CTAs that can be resident at once (cached per kernel and
// device); the pair kernel is persistent over that many pairs.
template <int BN, bool BW, bool I8 = false>
int pair_clusters() {
  static std::atomic<int> cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 0;
  if (cache[dev].load(std::memory_order_relaxed) == 0) {
    using C = Cfg2<BN, BW>;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * static_cast<unsigned>(num_sms()));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<BN, BW, I8>, &cfg) != cudaSuccess) n = 0;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return cache[dev].load(std::memory_order_relaxed);
}

template <int BN, bool BW, bool I8 = false>
fp8q_status launch_pair(const void* a_op, const void* b_op, const GemmArgs& p, cudaStream_t stream) {
  using C = Cfg2<BN, BW>;
  CUtensorMap ma, mb;
  if (!tensor_map(a_op, p.rows_a, p.K, BM, &ma) || !tensor_map(b_op, p.rows_b, p.K, C::HB, &mb))
    return FP8Q_ERR_CUDA;
  static std::atomic<int> attr_done[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(gemm_pair_kernel<BN, BW, I8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return FP8Q_ERR_CUDA;
    attr_done[dev].store(1, std::memory_order_relaxed);
  }
  const int nc = pair_clusters<BN, BW, I8>();
  if (nc < 1) return FP8Q_ERR_UNSUPPORTED;
  const int npairs = p.units < nc ? p.units : nc;
  return launch_kernel(gemm_pair_kernel<BN, BW, I8>, dim3(2 * static_cast<unsigned>(npairs)),
                       dim3(C::THREADS), C::SMEM_BYTES, stream, 2, ma, mb, p);
}

// ---------------------------------------------------------------- dispatch

std::mutex g_force_mu;
bool g_forced = false;
fp8q_gemm_variant g_force{0, 1, 128, 0};

// blockwise: 0 per-token / per-channel scales, 1 fp32 block scales, 2 E8M0
// block scales (block-scaled MMA).
bool variant_supported(const fp8q_gemm_variant& v, int blockwise) {
  if (v.cta_pair != 0 && v.cta_pair != 1) return false;
  // warp-MMA weight streaming for M <= 8 (fp32 scales, per token or blockwise)
  if (v.block_n == kDecodeMaxM) return blockwise <= 1 && v.swap_ab == 1 && v.split_k == 1 && !v.cta_pair;
  if (blockwise == 3) blockwise = 0;   // int8: the per-token scheme's variants
  if (blockwise == 2) {
    // single CTAs only; 224- and 256-column tiles (one accumulator buffer at 256)
    if (v.cta_pair || v.split_k < 0 || v.split_k > 64) return false;
    if (v.swap_ab) return v.block_n == 16 || v.block_n == 32 || v.block_n == 64 || v.block_n == 128;
    return v.block_n == 128 || v.block_n == 224 || v.block_n == 256;
  }
  // (pairs: blockwise with 128-column tiles -- four accumulator buffers --,
  // per token with 128 or 256)
  if (v.cta_pair) return !v.swap_ab && v.split_k == 1 && (v.block_n == 128 || (!blockwise && v.block_n == 256));
  if (v.split_k < 0 || v.split_k > 64) return false;   // 0: stream-K
  if (v.swap_ab) return v.block_n == 16 || v.block_n == 32 || v.block_n == 64 || v.block_n == 128;
  if (blockwise) return v.block_n == 128 || v.block_n == 256;
  return v.block_n == 128 || v.block_n == 256;
}

int epi_warps(const fp8q_gemm_variant& v, int blockwise) {
  if (blockwise == 2 || blockwise == 3) return 4;
  if (v.cta_pair) return blockwise ? (v.block_n >= 256 ? 16 : 8) : 4;
  return (blockwise && v.block_n >= 128) ? 8 : 4;
}

// Measured variant table: for each (scheme, N, K) the fastest variant per
// bucket of M, timed on a B200 by tune.py (which writes the included file).
// A row applies to m_prev < M <= m_max, m_prev being the next smaller m_max
// of the same (scheme, N, K); M above the largest bucket takes that bucket.
struct TunedVariant {
  int blockwise;
  int64_t m_max, n, k;
  int swap_ab, split_k, block_n, cta_pair;
};
constexpr TunedVariant kTuned[] = {
#include "fp8q_variant_table.inc"
    {-1, 0, 0, 0, 0, 0, 0, 0},   // end marker
};

bool tuned_variant(int64_t M, int64_t N, int64_t K, int blockwise, fp8q_gemm_variant* out) {
  const TunedVariant* best = nullptr;   // smallest m_max >= M
  const TunedVariant* top = nullptr;    // largest m_max
  for (const TunedVariant& t : kTuned) {
    if (t.blockwise != blockwise || t.n != N || t.k != K) continue;
    if (t.m_max >= M && (!best || t.m_max < best->m_max)) best = &t;
    if (!top || t.m_max > top->m_max) top = &t;
  }
  if (!best) best = top;
  if (!best) return false;
  out->swap_ab = best->swap_ab;
  out->split_k = best->split_k;
  out->block_n = best->block_n;
  out->cta_pair = best->cta_pair;
  return variant_supported(*out, blockwise);
}

// Shapes outside the table: rules drawn from the same measurements.
fp8q_gemm_variant heuristic_variant(int64_t M, int64_t N, int64_t K, int blockwise,
                                    bool allow_decode = true) {
  fp8q_gemm_variant v;
  v.cta_pair = 0;
  // M <= 8: the warp-MMA weight streaming kernel, measured fastest on every
  // table shape with K <= 12288 (the longer K of a 25600-deep layer leaves its
  // warps too few loads in flight; there Swap-AB tiles stay faster)
  if (allow_decode && blockwise <= 1 && M <= kDecodeMaxM && K % BK == 0 && N % kDecodeRows == 0 &&
      K <= 16384) {
    v.swap_ab = 1;
    v.split_k = 1;
    v.block_n = kDecodeMaxM;
    return v;
  }
  if (M <= 128) {
    // Swap-AB: the weight rows fill the 128-row MMA slot, the tokens its N.
    v.swap_ab = 1;
    v.block_n = M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
  } else {
    v.swap_ab = 0;
    v.block_n = 256;
  }
  const int64_t rows_a = v.swap_ab ? N : M, rows_b = v.swap_ab ? M : N;
  const int64_t tiles = ((rows_a + BM - 1) / BM) * ((rows_b + v.block_n - 1) / v.block_n);
  const int64_t kblocks = (K + BK - 1) / BK;
  const int64_t sms = num_sms();
  // Per-token scales from M = 512 up: 256x256 tiles on CTA pairs once there
  // are at least 40 of them (the measured table picks them for every layer
  // shape from M = 512 or 1024 on; fewer tiles leave too many SMs idle).
  const int64_t pair_tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + 255) / 256);
  if (!blockwise && M >= 512 && pair_tiles >= 40) {
    v.block_n = 256;
    v.split_k = 1;
    v.cta_pair = 1;
    return v;
  }
  if (tiles >= sms) {
    v.split_k = 1;
  } else if (blockwise && M > 16) {
    // The per-K-block promotion makes each SM's share of the K loop the
    // limit: stream-K spreads the K blocks over every SM.
    v.split_k = 0;
  } else {
    // Whole K ranges: as many per tile as fit on the SMs in one wave,
    // each at least 8 K blocks long.
    int64_t s = sms / tiles;
    if (s > kblocks / 8) s = kblocks / 8;
    v.split_k = static_cast<int>(s < 1 ? 1 : s);
  }
  return v;
}

fp8q_gemm_variant auto_variant(int64_t M, int64_t N, int64_t K, int blockwise) {
  fp8q_gemm_variant v;
  if (tuned_variant(M, N, K, blockwise, &v)) return v;
  return heuristic_variant(M, N, K, blockwise);
}

fp8q_gemm_variant pick_variant(int64_t M, int64_t N, int64_t K, int blockwise,
                               bool* forced = nullptr) {
  {
    std::lock_guard<std::mutex> lock(g_force_mu);
    if (forced) *forced = g_forced;
    if (g_forced) return g_force;
  }
  if (blockwise >= 2) {
    // int8 (3) and the block-scaled MMA (2) keep the whole K loop in TMEM like
    // the per-token kernel, so they follow the per-token scheme's measured
    // choice -- except its warp-MMA decode kernel (fp8 with fp32 scales only),
    // for which they take the tcgen05 rule's Swap-AB tiles.
    fp8q_gemm_variant v = auto_variant(M, N, K, 0);
    if (v.block_n == kDecodeMaxM) v = heuristic_variant(M, N, K, 0, false);
    if (blockwise == 3) return v;
    // E8M0: single CTAs (a CTA-pair choice becomes 128x256 single-CTA tiles)
    if (v.cta_pair) v = fp8q_gemm_variant{0, 1, 256, 0};
    return v;
  }
  return auto_variant(M, N, K, blockwise);
}

struct Plan {
  fp8q_gemm_variant v;
  int tiles_a, tiles_b, kblocks, split, kb_per_split, units;
  int streamk, seg_len, total_iters, grid, max_contrib;
  size_t counter_bytes, ws_bytes;
};

Plan make_plan(int64_t M, int64_t N, int64_t K, int blockwise, const fp8q_gemm_variant& v) {
  Plan pl;
  pl.v = v;
  const int64_t rows_a = v.swap_ab ? N : M, rows_b = v.swap_ab ? M : N;
  const int tile_rows = v.cta_pair ? 2 * BM : BM;      // CTA pairs: 256-row tiles
  pl.tiles_a = static_cast<int>((rows_a + tile_rows - 1) / tile_rows);
  pl.tiles_b = static_cast<int>((rows_b + v.block_n - 1) / v.block_n);
  pl.kblocks = static_cast<int>((K + BK - 1) / BK);
  const int64_t tiles = static_cast<int64_t>(pl.tiles_a) * pl.tiles_b;
  pl.streamk = 0;
  pl.seg_len = 0;
  pl.total_iters = 0;
  if (v.cta_pair) {
    pl.split = 1;
    pl.kb_per_split = pl.kblocks;
    pl.units = static_cast<int>(tiles);
    pl.grid = 0;
    pl.max_contrib = 1;
  } else if (v.split_k == 0) {
    // stream-K: equal K-block ranges over at most one CTA per SM
    const int64_t total = tiles * pl.kblocks;
    int64_t grid = num_sms();
    if (grid > total) grid = total;
    pl.streamk = 1;
    pl.total_iters = static_cast<int>(total);
    pl.seg_len = static_cast<int>((total + grid - 1) / grid);
    pl.grid = static_cast<int>((total + pl.seg_len - 1) / pl.seg_len);
    pl.max_contrib = (pl.kblocks + pl.seg_len - 1) / pl.seg_len + 1;
    if (pl.max_contrib > pl.grid) pl.max_contrib = pl.grid;
    pl.split = 1;
    pl.kb_per_split = pl.kblocks;
    pl.units = 0;
  } else {
    int split = v.split_k < pl.kblocks ? v.split_k : pl.kblocks;
    if (split < 1) split = 1;
    pl.kb_per_split = (pl.kblocks + split - 1) / split;
    pl.split = (pl.kblocks + pl.kb_per_split - 1) / pl.kb_per_split;   // every split non-empty
    pl.units = static_cast<int>(tiles * pl.split);
    pl.grid = pl.units < num_sms() ? pl.units : num_sms();
    pl.max_contrib = pl.split;
  }
  if (pl.max_contrib > 1) {
    pl.counter_bytes = ((static_cast<size_t>(tiles) * epi_warps(v, blockwise) * sizeof(int) + 255) / 256) * 256;
    pl.ws_bytes = pl.counter_bytes + static_cast<size_t>(tiles) * pl.max_contrib * BM * v.block_n * sizeof(float);
  } else {
    pl.counter_bytes = 0;
    pl.ws_bytes = 0;
  }
  return pl;
}

template <bool BW>
fp8q_status launch_decode(const void* a_q, const void* b_q, const GemmArgs& p, cudaStream_t stream) {
  if (p.M > kDecodeMaxM || p.K % BK != 0 || p.N % kDecodeRows != 0) return FP8Q_ERR_UNSUPPORTED;
  return launch_kernel(decode_kernel<BW>, dim3(static_cast<unsigned>(p.N / kDecodeRows)),
                       dim3(32 * kDecodeWarps), 0, stream, 1, static_cast<const uint8_t*>(a_q),
                       static_cast<const uint8_t*>(b_q), p);
}

template <bool BW, bool MX = false, bool I8 = false>
fp8q_status run_gemm(const void* a_q, const void* b_q, GemmArgs& p, const Plan& pl, void* ws,
                     cudaStream_t stream) {
  p.tiles_a = pl.tiles_a;
  p.tiles_b = pl.tiles_b;
  p.kblocks = pl.kblocks;
  p.split = pl.split;
  p.kb_per_split = pl.kb_per_split;
  p.units = pl.units;
  p.streamk = pl.streamk;
  p.seg_len = pl.seg_len;
  p.total_iters = pl.total_iters;
  p.max_contrib = pl.max_contrib;
  p.counters = pl.max_contrib > 1 ? static_cast<int*>(ws) : nullptr;
  p.ws = pl.max_contrib > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.counter_bytes) : nullptr;
  p.status = device_status_ptr();
  const int bn = pl.v.block_n;
  if (bn == kDecodeMaxM) {
    if constexpr (MX || I8) return FP8Q_ERR_UNSUPPORTED;
    else return launch_decode<BW>(a_q, b_q, p, stream);
  }
  if constexpr (MX) {
    if (pl.v.cta_pair) return FP8Q_ERR_UNSUPPORTED;
    if (pl.v.swap_ab) {
      p.rows_a = p.N;
      p.rows_b = p.M;
      switch (bn) {
        case 16: return launch_gemm<16, true, false, true>(b_q, a_q, p, stream);
        case 32: return launch_gemm<32, true, false, true>(b_q, a_q, p, stream);
        case 64: return launch_gemm<64, true, false, true>(b_q, a_q, p, stream);
        case 128: return launch_gemm<128, true, false, true>(b_q, a_q, p, stream);
        default: return FP8Q_ERR_UNSUPPORTED;
      }
    }
    p.rows_a = p.M;
    p.rows_b = p.N;
    if (bn == 128) return launch_gemm<128, false, false, true>(a_q, b_q, p, stream);
    if (bn == 224) return launch_gemm<224, false, false, true>(a_q, b_q, p, stream);
    if (bn == 256) return launch_gemm<256, false, false, true>(a_q, b_q, p, stream);
    return FP8Q_ERR_UNSUPPORTED;
  }
  if (pl.v.cta_pair) {
    p.rows_a = p.M;
    p.rows_b = p.N;
    if (bn == 128) return launch_pair<128, BW, I8>(a_q, b_q, p, stream);
    if constexpr (!BW) {
      if (bn == 256) return launch_pair<256, false, I8>(a_q, b_q, p, stream);
    }
    return FP8Q_ERR_UNSUPPORTED;
  }
  if (pl.v.swap_ab) {
    p.rows_a = p.N;
    p.rows_b = p.M;
    switch (bn) {
      case 16: return launch_gemm<16, true, BW, false, I8>(b_q, a_q, p, stream);
      case 32: return launch_gemm<32, true, BW, false, I8>(b_q, a_q, p, stream);
      case 64: return launch_gemm<64, true, BW, false, I8>(b_q, a_q, p, stream);
      case 128: return launch_gemm<128, true, BW, false, I8>(b_q, a_q, p, stream);
      default: return FP8Q_ERR_UNSUPPORTED;
    }
  }
  p.rows_a = p.M;
  p.rows_b = p.N;
  if (bn == 128) return launch_gemm<128, false, BW, false, I8>(a_q, b_q, p, stream);
  if (bn == 256) return launch_gemm<256, false, BW, false, I8>(a_q, b_q, p, stream);
  return FP8Q_ERR_UNSUPPORTED;
}

constexpr int64_t kMaxDim = (1LL << 31) - 512;

fp8q_status check_gemm(const void* a_q, const void* b_q, const void* sa, const void* sb,
                       int64_t M, int64_t N, int64_t K, const void* y, int64_t ldy) {
  if (M < 0 || N <= 0 || K <= 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
    return FP8Q_ERR_INVALID_ARG;
  if (N % 16 != 0 || K % 16 != 0) return FP8Q_ERR_INVALID_ARG;
  if (ldy < N || ldy % 8 != 0) return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;  // nothing is read or written: pointers may be null
  if (!a_q || !b_q || !sa || !sb || !y) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(a_q, 16) || !aligned(b_q, 16) || !aligned(y, 16) || !aligned(sa, 4) ||
      !aligned(sb, 4))
    return FP8Q_ERR_INVALID_ARG;
  return FP8Q_OK;
}

// The blockwise kernels address activation scales with 32-bit element
// offsets (m * as_stride_m + kb * as_stride_kb, kb running a few blocks past
// the last one): every such offset must stay below 2^31.
bool scale_offsets_fit(int64_t M, int64_t K, int64_t as_stride_m, int64_t as_stride_kb) {
  const int64_t last = (M - 1) * as_stride_m + (K / 128 + 8) * as_stride_kb;
  return last < (1LL << 31);
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" fp8q_status fp8q_select_gemm_variant(int64_t M, int64_t N, int64_t K, int blockwise,
                                                fp8q_gemm_variant* out) {
  if (!out || M < 0 || N <= 0 || K <= 0) return FP8Q_ERR_INVALID_ARG;
  *out = pick_variant(M, N, K, blockwise);
  const Plan pl = make_plan(M, N, K, blockwise, *out);
  out->split_k = pl.streamk ? 0 : pl.split;
  return FP8Q_OK;
}

extern "C" fp8q_status fp8q_force_gemm_variant(const fp8q_gemm_variant* v) {
  std::lock_guard<std::mutex> lock(g_force_mu);
  if (!v) {
    g_forced = false;
    return FP8Q_OK;
  }
  if (!variant_supported(*v, 0) && !variant_supported(*v, 1) && !variant_supported(*v, 2))
    return FP8Q_ERR_INVALID_ARG;
  g_force = *v;
  g_forced = true;
  return FP8Q_OK;
}

extern "C" size_t fp8q_workspace_bytes(int64_t M, int64_t N, int64_t K, int blockwise) {
  if (M <= 0 || N <= 0 || K <= 0 || blockwise < 0 || blockwise > 3) return 0;
  const fp8q_gemm_variant v = pick_variant(M, N, K, blockwise);
  return make_plan(M, N, K, blockwise, v).ws_bytes;
}

extern "C" fp8q_status fp8q_scaled_mm(const void* a_q, const void* b_q, const float* a_scale,
                                      int a_per_token, const float* b_scale, int b_per_channel,
                                      int64_t M, int64_t N, int64_t K, void* y, int64_t ldy,
                                      void* workspace, size_t ws_bytes, void* stream) {
  fp8q_status st = check_gemm(a_q, b_q, a_scale, b_scale, M, N, K, y, ldy);
  if (st != FP8Q_OK) return st;
  if ((a_per_token != 0 && a_per_token != 1) || (b_per_channel != 0 && b_per_channel != 1))
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  const fp8q_gemm_variant v = pick_variant(M, N, K, 0);
  if (!variant_supported(v, 0)) return FP8Q_ERR_UNSUPPORTED;
  const Plan pl = make_plan(M, N, K, 0, v);
  if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes || !aligned(workspace, 256)))
    return FP8Q_ERR_INVALID_ARG;
  GemmArgs p{};
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.sa = a_scale;
  p.sa_sm = a_per_token ? 1 : 0;
  p.sa_skb = 0;
  p.sb = b_scale;
  p.sb_sn = b_per_channel ? 1 : 0;
  p.sb_snb = 0;
  p.sb_skb = 0;
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  return run_gemm<false>(a_q, b_q, p, pl, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_scaled_mm_blockwise(const void* a_q, const void* b_q,
                                                const float* a_scale, int64_t as_stride_m,
                                                int64_t as_stride_kb, const float* b_scale,
                                                int64_t M, int64_t N, int64_t K, void* y,
                                                int64_t ldy, void* workspace, size_t ws_bytes,
                                                void* stream) {
  fp8q_status st = check_gemm(a_q, b_q, a_scale, b_scale, M, N, K, y, ldy);
  if (st != FP8Q_OK) return st;
  if (N % 128 != 0 || K % 128 != 0 || as_stride_m < 0 || as_stride_kb < 0)
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!scale_offsets_fit(M, K, as_stride_m, as_stride_kb)) return FP8Q_ERR_INVALID_ARG;
  const fp8q_gemm_variant v = pick_variant(M, N, K, 1);
  if (!variant_supported(v, 1)) return FP8Q_ERR_UNSUPPORTED;
  const Plan pl = make_plan(M, N, K, 1, v);
  if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes || !aligned(workspace, 256)))
    return FP8Q_ERR_INVALID_ARG;
  GemmArgs p{};
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.sa = a_scale;
  p.sa_sm = as_stride_m;
  p.sa_skb = as_stride_kb;
  p.sb = b_scale;
  p.sb_sn = 0;
  p.sb_snb = K / 128;
  p.sb_skb = 1;
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  return run_gemm<true>(a_q, b_q, p, pl, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_scaled_mm_i8(const void* a_q, const void* b_q, const float* a_scale,
                                         int a_per_token, const float* b_scale, int b_per_channel,
                                         int64_t M, int64_t N, int64_t K, void* y, int64_t ldy,
                                         void* workspace, size_t ws_bytes, void* stream) {
  fp8q_status st = check_gemm(a_q, b_q, a_scale, b_scale, M, N, K, y, ldy);
  if (st != FP8Q_OK) return st;
  if ((a_per_token != 0 && a_per_token != 1) || (b_per_channel != 0 && b_per_channel != 1))
    return FP8Q_ERR_INVALID_ARG;
  if (K > 133152) return FP8Q_ERR_INVALID_ARG;   // 128^2 K must stay below 2^31
  if (M == 0) return FP8Q_OK;
  const fp8q_gemm_variant v = pick_variant(M, N, K, 3);
  if (!variant_supported(v, 3)) return FP8Q_ERR_UNSUPPORTED;
  const Plan pl = make_plan(M, N, K, 3, v);
  if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes || !aligned(workspace, 256)))
    return FP8Q_ERR_INVALID_ARG;
  GemmArgs p{};
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.sa = a_scale;
  p.sa_sm = a_per_token ? 1 : 0;
  p.sb = b_scale;
  p.sb_sn = b_per_channel ? 1 : 0;
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  return run_gemm<false, false, true>(a_q, b_q, p, pl, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_scaled_mm_blockwise_e8m0(const void* a_q, const void* b_q,
                                                     const uint8_t* a_sf, int64_t as_stride_m,
                                                     int64_t as_stride_kb, const uint8_t* b_sf,
                                                     int64_t M, int64_t N, int64_t K, void* y,
                                                     int64_t ldy, void* workspace, size_t ws_bytes,
                                                     void* stream) {
  if (M < 0 || N <= 0 || K <= 0 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
    return FP8Q_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % 128 != 0 || ldy < N || ldy % 8 != 0 || as_stride_m < 0 || as_stride_kb < 0)
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!a_q || !b_q || !a_sf || !b_sf || !y) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(a_q, 16) || !aligned(b_q, 16) || !aligned(y, 16)) return FP8Q_ERR_INVALID_ARG;
  if (!scale_offsets_fit(M, K, as_stride_m, as_stride_kb)) return FP8Q_ERR_INVALID_ARG;
  const fp8q_gemm_variant v = pick_variant(M, N, K, 2);
  if (!variant_supported(v, 2)) return FP8Q_ERR_UNSUPPORTED;
  const Plan pl = make_plan(M, N, K, 2, v);
  if (pl.ws_bytes > 0 && (!workspace || ws_bytes < pl.ws_bytes || !aligned(workspace, 256)))
    return FP8Q_ERR_INVALID_ARG;
  GemmArgs p{};
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.sfa = a_sf;
  p.sfa_sm = as_stride_m;
  p.sfa_skb = as_stride_kb;
  p.sfb = b_sf;
  p.sfb_snb = K / 128;
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  return run_gemm<false, true>(a_q, b_q, p, pl, workspace, static_cast<cudaStream_t>(stream));
}

extern "C" fp8q_status fp8q_scaled_mm_blockwise_silu_quant(
    const void* a_q, const void* b_q, const float* a_scale, int64_t as_stride_m, int64_t as_stride_kb,
    const float* b_scale, int64_t M, int64_t N2, int64_t K, int ue8m0, void* q, int64_t ldq,
    float* scales, int64_t s_stride_m, int64_t s_stride_g, void* stream) {
  if (M < 0 || N2 <= 0 || K <= 0 || M > kMaxDim || N2 > kMaxDim || K > kMaxDim) return FP8Q_ERR_INVALID_ARG;
  if (N2 % 256 != 0 || K % 128 != 0 || as_stride_m < 0 || as_stride_kb < 0) return FP8Q_ERR_INVALID_ARG;
  if (ue8m0 < 0 || ue8m0 > 2 || s_stride_m < 0 || s_stride_g < 0 || ldq < N2 / 2 || ldq % 16 != 0)
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!a_q || !b_q || !a_scale || !b_scale || !q || !scales) return FP8Q_ERR_INVALID_ARG;
  if (!aligned(a_q, 16) || !aligned(b_q, 16) || !aligned(q, 16) || !aligned(a_scale, 4) ||
      !aligned(b_scale, 4) || !aligned(scales, ue8m0 == 2 ? 1 : 4))
    return FP8Q_ERR_INVALID_ARG;
  if (!scale_offsets_fit(M, K, as_stride_m, as_stride_kb)) return FP8Q_ERR_INVALID_ARG;
  // 128x256 single-CTA tiles over the whole K range (the epilogue needs the
  // finished sums); a forced variant does not apply here.
  const fp8q_gemm_variant v{0, 1, 256, 0};
  const Plan pl = make_plan(M, N2, K, 1, v);
  GemmArgs p{};
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N2);
  p.sa = a_scale;
  p.sa_sm = as_stride_m;
  p.sa_skb = as_stride_kb;
  p.sb = b_scale;
  p.sb_sn = 0;
  p.sb_snb = K / 128;
  p.sb_skb = 1;
  p.sq_q = static_cast<uint8_t*>(q);
  p.sq_ldq = ldq;
  p.sq_s = scales;
  p.sq_s_sm = s_stride_m;
  p.sq_s_sg = s_stride_g;
  p.sq_ue8m0 = ue8m0;
  p.sq_exact = fp8q_get_fused_quant_exact();
  p.tiles_a = pl.tiles_a;
  p.tiles_b = pl.tiles_b;
  p.kblocks = pl.kblocks;
  p.split = 1;
  p.kb_per_split = pl.kblocks;
  p.units = pl.units;
  p.max_contrib = 1;
  p.status = device_status_ptr();
  p.rows_a = p.M;
  p.rows_b = p.N;
  return launch_gemm<256, false, true, false, false, true>(a_q, b_q, p, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ no-allocation path
// Split-K scratch of fp8q_scaled_mm_blockwise_noalloc: one fixed device array,
// shared by every call on a device, so the call allocates nothing.  Host code
// must not pass the symbol itself to a kernel (on the host it names a
// stand-in, not device memory): its device address comes from
// cudaGetSymbolAddress, looked up once per device.
namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[FP8Q_NOALLOC_SCRATCH_BYTES];

void* noalloc_scratch_ptr() {
  static std::mutex mu;
  static void* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    cache[dev] = p;
  }
  return cache[dev];
}
}  // namespace

extern "C" fp8q_status fp8q_scaled_mm_blockwise_noalloc(const void* a_q, const void* b_q,
                                                        const float* a_scale, int64_t as_stride_m,
                                                        int64_t as_stride_kb, const float* b_scale,
                                                        int64_t M, int64_t N, int64_t K, void* y,
                                                        int64_t ldy, void* stream) {
  fp8q_status st = check_gemm(a_q, b_q, a_scale, b_scale, M, N, K, y, ldy);
  if (st != FP8Q_OK) return st;
  if (N % 128 != 0 || K % 128 != 0 || as_stride_m < 0 || as_stride_kb < 0)
    return FP8Q_ERR_INVALID_ARG;
  if (M == 0) return FP8Q_OK;
  if (!scale_offsets_fit(M, K, as_stride_m, as_stride_kb)) return FP8Q_ERR_INVALID_ARG;
  bool forced = false;
  fp8q_gemm_variant v = pick_variant(M, N, K, 1, &forced);
  if (!variant_supported(v, 1)) return FP8Q_ERR_UNSUPPORTED;
  Plan pl = make_plan(M, N, K, 1, v);
  if (pl.ws_bytes > FP8Q_NOALLOC_SCRATCH_BYTES && !forced) {
    // The chosen split's partials do not fit the fixed array; whole-K tiles
    // need no scratch at all.
    v.split_k = 1;
    pl = make_plan(M, N, K, 1, v);
  }
  if (pl.ws_bytes > FP8Q_NOALLOC_SCRATCH_BYTES) return FP8Q_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pl.ws_bytes > 0) {
    scratch = noalloc_scratch_ptr();
    if (!scratch) return FP8Q_ERR_CUDA;
    if (cudaMemsetAsync(scratch, 0, pl.counter_bytes, s) != cudaSuccess) return FP8Q_ERR_CUDA;
  }
  GemmArgs p{};
  p.K = static_cast<int>(K);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.sa = a_scale;
  p.sa_sm = as_stride_m;
  p.sa_skb = as_stride_kb;
  p.sb = b_scale;
  p.sb_sn = 0;
  p.sb_snb = K / 128;
  p.sb_skb = 1;
  p.y = static_cast<uint16_t*>(y);
  p.ldy = ldy;
  return run_gemm<true>(a_q, b_q, p, pl, scratch, s);
}
