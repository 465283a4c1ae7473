/*
 * fp8q.h -- C ABI of libfp8q, the B200 (sm_100a) FP8 W8A8 linear-layer path:
 * dynamic activation quantization fused with its producer, and the scaled FP8
 * GEMMs it feeds.
 *
 * The ops are the ones listed in "Helion in vLLM" (24-ai.news), section
 * "Kernels integrated into vLLM": items 1-3 and 5-7 (quantization) and 8-9
 * (GEMMs).  The pages name them but do not write out their arithmetic; this
 * library fixes it as follows.
 *
 *   scale      s = fl32(max(amax, 1e-10) / 448), amax = max |y| over the group
 *   UE8M0      (ue8m0 = 1) s is rounded up to the next power of two (a power of
 *              two is kept); the scale is still stored as fp32.  (ue8m0 = 2)
 *              the same power-of-two scale stored packed as one E8M0 byte:
 *              its biased exponent b, s = 2^(b - 127)
 *   codes      q = e4m3fn(fl32(y / s)), IEEE fp32 division, round to nearest
 *              even, saturating to +-448; the sign of zero is kept
 *   groups     contiguous 1x128 chunks of a row (group_size = 128), or the
 *              whole row (group_size = row length: "per token")
 *   y          the value quantized: x itself (group quant); bf16(bf16(x*r)*w)
 *              with r = 1/sqrt(mean(x^2)+eps) (RMSNorm); bf16(silu(g)*u)
 *              (SiLU*mul) -- one round-to-nearest-even to bf16 at each step
 *   GEMM       y[m,n] = bf16_rn(sum_k (qa[m,k] sa)(qb[n,k] sb)), fp32 accumulate
 *
 * Conventions shared by every entry point.
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *     library allocates no device memory in any call: scratch space is the
 *     caller's `workspace` (sized by fp8q_workspace_bytes).
 *   - bf16 tensors are raw IEEE bfloat16 bit patterns; codes are float8
 *     e4m3fn bytes; scales are fp32.  Matrices are row-major with a leading
 *     dimension `ld*` given in ELEMENTS.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous: they enqueue kernels and return; no
 *     call synchronizes the host except fp8q_last_device_status.  Calls can
 *     be captured into CUDA graphs.
 *   - Kernels are launched with programmatic dependent launch: one may begin
 *     its setup while the previous kernel on the stream is still running, but
 *     reads and writes nothing until that kernel has completed and its writes
 *     are visible.  The one early access is an L2 prefetch of a GEMM's first
 *     weight tiles, a cache hint with no visible effect (the data are read
 *     again after the wait), so stream order holds for every buffer.  Setting
 *     the environment variable FP8Q_PDL=0 before the first call launches
 *     kernels without it.
 *   - Argument errors are found on the host before anything is launched; the
 *     call then returns FP8Q_ERR_INVALID_ARG (or FP8Q_ERR_UNSUPPORTED) and
 *     launches nothing.  A launch failure returns FP8Q_ERR_CUDA.  A GEMM
 *     whose internal pipeline wait runs past its time limit (about one
 *     second) stops, records FP8Q_ERR_TIMEOUT in a device status word and
 *     returns; read it with fp8q_last_device_status.  No C++ exception
 *     crosses this interface.
 *   - Pointers to bf16 / code tensors must be 16-byte aligned; fp32 scale
 *     pointers 4-byte aligned (E8M0 byte arrays need no alignment).  With M = 0 a call validates its sizes and returns
 *     FP8Q_OK without touching memory; its pointers may then be NULL.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8Q_API __attribute__((visibility("default")))
#else
#define FP8Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8Q_OK = 0,
    FP8Q_ERR_INVALID_ARG = 1,  /* null pointer, bad size, stride or alignment */
    FP8Q_ERR_UNSUPPORTED = 2,  /* valid request this build does not handle    */
    FP8Q_ERR_CUDA = 3,         /* a CUDA runtime / driver call failed          */
    FP8Q_ERR_TIMEOUT = 4       /* a device-side wait gave up (device status)   */
} fp8q_status;

/* ------------------------------------------------------------------------ */
/* Activation quantization                                                   */
/* ------------------------------------------------------------------------ */

/*
 * fp8q_group_quant -- per_token_group_fp8_quant (group_size = 128) and
 * dynamic_per_token_scaled_fp8_quant (group_size = K) ("Helion in vLLM",
 * "Kernels integrated into vLLM", items 5 and 1).  Also quantizes weights per
 * output channel: a row of W [N, K] is one channel.
 *
 *   x        bf16 [M, K], leading dimension ldx (>= K, multiple of 8)
 *   M, K     M >= 0 (M = 0 is a no-op), K > 0 and a multiple of 16
 *   group_size  128 (K must then be a multiple of 128) or K
 *   ue8m0    0: fp32 scales; 1: scales rounded up to powers of two, fp32;
 *            2: the same power-of-two scales as packed E8M0 bytes -- `scales`
 *            then points to uint8 storage (any alignment) and the strides
 *            count bytes (the layout fp8q_scaled_mm_blockwise_e8m0 reads)
 *   q        e4m3 codes [M, K], leading dimension ldq (>= K, multiple of 16)
 *   scales   fp32 (or E8M0 bytes), scale of group g of row m at
 *            scales[m*s_stride_m + g*s_stride_g]
 *            (row-major [M, K/group]: s_stride_m = K/group, s_stride_g = 1;
 *            group-major [K/group, M]: s_stride_m = 1, s_stride_g = M)
 */
FP8Q_API fp8q_status fp8q_group_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int group_size,
                             int ue8m0, void* q, int64_t ldq, float* scales,
                             int64_t s_stride_m, int64_t s_stride_g, void* stream);

/*
 * fp8q_rmsnorm_quant -- rms_norm_dynamic_per_token_quant (group_size = H)
 * and rms_norm_per_block_quant (group_size = 128) ("Helion in vLLM",
 * "Kernels integrated into vLLM", items 2 and 6).  The norm is taken over the
 * whole row of H elements; the scales per group.
 *   y = bf16(bf16(x * r) * w),  r = 1 / sqrt(sum(x^2)/H + eps)
 *
 *   x [M, H] bf16 (ldx), w [H] bf16, eps >= 0; other arguments as in
 *   fp8q_group_quant with K = H.
 */
FP8Q_API fp8q_status fp8q_rmsnorm_quant(const void* x, const void* w, float eps, int64_t M, int64_t H,
                               int64_t ldx, int group_size, int ue8m0, void* q, int64_t ldq,
                               float* scales, int64_t s_stride_m, int64_t s_stride_g,
                               void* stream);

/*
 * fp8q_add_rmsnorm_quant -- residual add fused into the RMSNorm quant, the
 * fusion "on either side of the path" that continues the pages' cut of the
 * call count by fused ops ("Helion in vLLM", "Kernels integrated into vLLM").
 *   h = bf16(x + residual)   (one rounding of the exact sum)
 *   residual <- h            (the residual stream is updated in place)
 *   q, scales = rmsnorm_quant(h)  exactly as fp8q_rmsnorm_quant
 * This is what the unfused chain (bf16 add, then fp8q_rmsnorm_quant) gives.
 *
 *   x [M, H] bf16 (ldx), residual [M, H] bf16 (ldr >= H, multiple of 8,
 *   16-byte aligned; read and written; must not overlap x, w, q or scales);
 *   other arguments as in fp8q_rmsnorm_quant.
 */
FP8Q_API fp8q_status fp8q_add_rmsnorm_quant(const void* x, void* residual, const void* w, float eps,
                                            int64_t M, int64_t H, int64_t ldx, int64_t ldr,
                                            int group_size, int ue8m0, void* q, int64_t ldq,
                                            float* scales, int64_t s_stride_m, int64_t s_stride_g,
                                            void* stream);

/*
 * fp8q_set_fused_quant_exact -- arithmetic of the producer-fused quant ops,
 * whose tolerance the pages' workload fixes at >= 99.9% of codes identical to
 * the definition, the rest within one step, scales within 1e-5 relative
 * ("Helion in vLLM", "Per-kernel performance": the fused ops are measured
 * against the unfused chain).
 *   exact = 0 (default): fp8q_silu_mul_quant and fp8q_silu_mul_quant_i8 with
 *     per-token scales compute y with fp32 ex2/rcp approximations, within one
 *     bf16 step of its definition and equal to it except next to a bf16
 *     rounding midpoint; the elements that can decide the row's amax are
 *     recomputed exactly, so every scale is bit-exact, and codes are the exact
 *     e4m3 (or int8) codes of fl32(y / s).  In the gate_up GEMM with the
 *     fused SiLU*mul quant (fp8q_scaled_mm_blockwise_silu_quant) a y whose
 *     rounding the fp32 bracket leaves open (about 1e-3 of the values) keeps
 *     the lower bracket end, within one bf16 step, unless it can decide its
 *     group's amax: scales stay bit-exact, codes differ only where such a y
 *     does.  All other fused ops (RMSNorm, residual add + RMSNorm, the
 *     standalone 1x128 SiLU*mul) are bit-exact in this mode too: a fast
 *     arithmetic measured no faster for them.
 *   exact = 1: every y is the correctly rounded value of its definition, so
 *     codes and scales of every fused op are bit-exact.
 * Process-wide; applies to calls made after it returns (captured CUDA graphs
 * keep the kernels they captured).  Other values: FP8Q_ERR_INVALID_ARG.
 * fp8q_get_fused_quant_exact returns the current setting.
 */
FP8Q_API fp8q_status fp8q_set_fused_quant_exact(int exact);
FP8Q_API int fp8q_get_fused_quant_exact(void);

/*
 * fp8q_silu_mul_quant -- silu_and_mul_dynamic_per_token_quant (group_size = I)
 * and silu_and_mul_per_block_quant (group_size = 128) ("Helion in vLLM",
 * "Kernels integrated into vLLM", items 3 and 7).
 *   row m of x is [gate (I) | up (I)];  y = bf16(silu(gate) * up),
 *   silu(t) = t / (1 + exp(-t))
 *
 *   x [M, 2I] bf16 (ldx >= 2I, multiple of 8); q [M, I] (ldq); other
 *   arguments as in fp8q_group_quant with K = I.
 */
FP8Q_API fp8q_status fp8q_silu_mul_quant(const void* x, int64_t M, int64_t I, int64_t ldx, int group_size,
                                int ue8m0, void* q, int64_t ldq, float* scales,
                                int64_t s_stride_m, int64_t s_stride_g, void* stream);

/*
 * fp8q_qk_norm_rope -- fused_qk_norm_rope ("Helion in vLLM" (24-ai.news),
 * "Kernels integrated into vLLM", item 4; its arguments as the vllm PR #44010
 * page lists them, section "Code analysis"), in place on the packed qkv
 * output of the qkv projection.  The pages print no arithmetic; this library
 * applies, to every q and k head of every token,
 *   the RMSNorm of this header:  r = 1/sqrt(mean(x^2) + eps),
 *                                y = bf16(bf16(x r) w)   (w = q or k weight)
 *   then the rotary embedding at p = positions[t], cos = cache[p][i],
 *   sin = cache[p][D/2 + i], on pairs (i, i + D/2) (is_neox = 1) or
 *   (2i, 2i + 1) (is_neox = 0):
 *                                a' = bf16(a cos - b sin), b' = bf16(b cos + a sin)
 * v heads are not touched.  Arithmetic is fp32 (the norm's reciprocal root to
 * about one fp32 ulp); results are the bf16 rounding of the definition
 * except where an fp32 result lies within a few fp32 ulps of a bf16 rounding
 * midpoint (then the neighbouring bf16 value).
 *
 *   qkv        bf16 [T, ld], row t = [q (hq heads) | k (hk) | v (hv)], head_dim D
 *              each; ld >= (hq + hk + hv) D, multiple of 8; 16-byte aligned
 *   head_dim   64, 128 or 256 (else FP8Q_ERR_UNSUPPORTED)
 *   q_weight, k_weight  bf16 [D]
 *   cos_sin_cache  fp32 [max_position, D]: D/2 cosines then D/2 sines per row
 *   positions  int64 [T], each in [0, max_position); a position outside it
 *              is not read: the token uses row 0 and the device status word
 *              records FP8Q_ERR_INVALID_ARG (see fp8q_last_device_status)
 */
FP8Q_API fp8q_status fp8q_qk_norm_rope(void* qkv, int64_t T, int64_t ld, int num_heads_q,
                                       int num_heads_k, int num_heads_v, int head_dim, float eps,
                                       const void* q_weight, const void* k_weight,
                                       const float* cos_sin_cache, int64_t max_position,
                                       const int64_t* positions, int is_neox, void* stream);

/* ------------------------------------------------------------------------ */
/* Scaled FP8 GEMMs                                                          */
/* ------------------------------------------------------------------------ */

/*
 * fp8q_scaled_mm -- scaled_mm ("Helion in vLLM", "Kernels integrated into
 * vLLM", item 8; the FP8_Dynamic scheme of "Helion linear backend"
 * (aihirek.info), section "Autotuning selects the variant").
 *   y[m, n] = bf16_rn( sa(m) * sb(n) * sum_k qa[m, k] * qb[n, k] )
 *
 *   a_q      e4m3 [M, K], rows contiguous (row stride K)
 *   b_q      e4m3 [N, K], rows contiguous (nn.Linear weight layout)
 *   a_scale  fp32: [M] if a_per_token else [1]
 *   b_scale  fp32: [N] if b_per_channel else [1]
 *   M >= 0 (M = 0 is a no-op), N > 0 a multiple of 16, K > 0 a multiple of 16
 *   y        bf16 [M, N], leading dimension ldy (>= N, multiple of 8)
 *   workspace / ws_bytes  device scratch of at least
 *            fp8q_workspace_bytes(M, N, K, 0) bytes (may be NULL when that
 *            is 0).  It must be zero-filled before its first use.  A call
 *            whose kernels finish normally leaves the part that must start
 *            at zero (the split-K arrival counters) at zero again, so the
 *            same workspace can be reused without clearing; after
 *            FP8Q_ERR_TIMEOUT, zero-fill it again.  Calls that share one
 *            workspace must not overlap in time.
 */
FP8Q_API fp8q_status fp8q_scaled_mm(const void* a_q, const void* b_q, const float* a_scale,
                           int a_per_token, const float* b_scale, int b_per_channel, int64_t M,
                           int64_t N, int64_t K, void* y, int64_t ldy, void* workspace,
                           size_t ws_bytes, void* stream);

/*
 * fp8q_scaled_mm_blockwise -- scaled_mm_blockwise ("Helion in vLLM",
 * "Kernels integrated into vLLM", item 9; the Block_FP8 scheme of "Helion
 * linear backend" (aihirek.info), section "Autotuning selects the variant").
 *   y[m, n] = bf16_rn( sum_kb sa[m, kb] * sb[n/128, kb] * P_kb[m, n] ),
 *   P_kb = fp32 sum over k in [128 kb, 128 kb + 128) of qa[m, k] * qb[n, k]
 *
 *   a_scale  fp32, one scale per 1x128 group of A: sa[m, kb] at
 *            a_scale[m*as_stride_m + kb*as_stride_kb]; strides >= 0 and
 *            (M-1)*as_stride_m + (K/128+8)*as_stride_kb < 2^31 (else
 *            FP8Q_ERR_INVALID_ARG; any scale array that fits in memory does)
 *   b_scale  fp32 [N/128, K/128] row-major, one scale per 128x128 block of B
 *   N and K multiples of 128; other arguments as in fp8q_scaled_mm, with
 *   fp8q_workspace_bytes(M, N, K, 1).
 */
FP8Q_API fp8q_status fp8q_scaled_mm_blockwise(const void* a_q, const void* b_q, const float* a_scale,
                                     int64_t as_stride_m, int64_t as_stride_kb,
                                     const float* b_scale, int64_t M, int64_t N, int64_t K,
                                     void* y, int64_t ldy, void* workspace, size_t ws_bytes,
                                     void* stream);

/*
 * fp8q_scaled_mm_blockwise_silu_quant -- the gate_up projection with the
 * SiLU*mul quant fused into its epilogue: one of the fusions "on either side
 * of the path" that continue the pages' cut of the call count ("Helion in
 * vLLM", "Kernels integrated into vLLM": fused ops replace chains of calls).
 * In the exact mode (fp8q_set_fused_quant_exact(1)) equal to, and
 * bit-identical with,
 *   h = fp8q_scaled_mm_blockwise(a, W)          (bf16 [M, 2I] = [gate | up])
 *   q, scales = fp8q_silu_mul_quant(h, group_size = 128, ue8m0)
 * run with the same 128x256 whole-K GEMM variant, without ever writing h; in
 * the fast mode (the default) the scales are the same and the codes meet the
 * fused-quant tolerance (see fp8q_set_fused_quant_exact).
 *
 *   b_q, b_scale  the gate_up weight [2I, K] and its [2I/128, K/128] block
 *            scales with the rows interleaved in 128-row blocks:
 *            [gate rows 0-127 | up rows 0-127 | gate 128-255 | up 128-255 | ...]
 *            (block row 2j = gate block j, 2j + 1 = up block j)
 *   N2       2I, a multiple of 256
 *   a_q, a_scale, as_stride_m, as_stride_kb, M, K   as in fp8q_scaled_mm_blockwise
 *   ue8m0, q [M, I] (ldq >= I, multiple of 16), scales, s_stride_m,
 *   s_stride_g   as in fp8q_silu_mul_quant with group_size 128
 * Runs 128x256 single-CTA tiles over the whole K range (no split-K and no
 * workspace; fp8q_force_gemm_variant does not apply).
 */
FP8Q_API fp8q_status fp8q_scaled_mm_blockwise_silu_quant(
    const void* a_q, const void* b_q, const float* a_scale, int64_t as_stride_m,
    int64_t as_stride_kb, const float* b_scale, int64_t M, int64_t N2, int64_t K, int ue8m0,
    void* q, int64_t ldq, float* scales, int64_t s_stride_m, int64_t s_stride_g, void* stream);

/*
 * fp8q_scaled_mm_blockwise_e8m0 -- scaled_mm_blockwise with power-of-two
 * block scales stored as E8M0 bytes, the form the pages say DeepGEMM needs
 * on B200 ("Helion in vLLM" (24-ai.news), section "Practical limits"; E8M0
 * block scales on SM100 in the MXFP4 CUTLASS MoE page, vllm PR #37463).
 *   y[m, n] = bf16_rn( sum_kb 2^(ea[m,kb]-127) 2^(eb[n/128,kb]-127) P_kb[m, n] )
 * The tensor core applies the scales itself (tcgen05.mma
 * kind::mxf8f6f4.block_scale, each 1x128 / 128x128 scale repeated over its
 * four 32-deep K slices), so the fp32 accumulator stays in TMEM for the whole
 * K range; the result equals fp8q_scaled_mm_blockwise on the decoded scales
 * up to fp32 summation order.
 *
 *   a_sf     uint8 E8M0, one byte per 1x128 group of A: ea[m, kb] at
 *            a_sf[m*as_stride_m + kb*as_stride_kb] (what fp8q_group_quant and
 *            the fused quant ops write with ue8m0 = 2); the offset rule of
 *            fp8q_scaled_mm_blockwise applies
 *   b_sf     uint8 E8M0 [N/128, K/128] row-major, one byte per 128x128 block
 *   A byte of 255 (E8M0 NaN) makes the affected outputs NaN.  N and K
 *   multiples of 128; other arguments as in fp8q_scaled_mm_blockwise, with
 *   fp8q_workspace_bytes(M, N, K, 2).  Variants: Swap-AB tiles (block_n
 *   16..128), or 128-row tiles of block_n 128, 224 (two accumulator buffers
 *   next to the scale factors in TMEM) or 256 (one buffer; the automatic
 *   choice for wide tiles); no CTA pairs.
 */
FP8Q_API fp8q_status fp8q_scaled_mm_blockwise_e8m0(const void* a_q, const void* b_q,
                                                   const uint8_t* a_sf, int64_t as_stride_m,
                                                   int64_t as_stride_kb, const uint8_t* b_sf,
                                                   int64_t M, int64_t N, int64_t K, void* y,
                                                   int64_t ldy, void* workspace, size_t ws_bytes,
                                                   void* stream);

/*
 * fp8q_scaled_mm_blockwise_noalloc -- the same GEMM as
 * fp8q_scaled_mm_blockwise, for callers that cannot hand the library any
 * device memory beyond their inputs and outputs.  (The pages have no
 * counterpart; this is a deployment convenience of this library.)
 *
 * Some callers cannot allocate: an inference engine that reserved all free
 * HBM for its KV cache at start-up, a plugin interface that gives a kernel
 * only its input and output buffers, or a latency-critical path where
 * cudaMalloc / cudaFree (which can synchronize the device) are not allowed.
 * This entry point allocates nothing.  Its split-K scratch is one fixed
 * device array of FP8Q_NOALLOC_SCRATCH_BYTES (16 MiB) inside the library,
 * which every GPU that loads the library holds until the process exits.
 *
 *   Arguments are those of fp8q_scaled_mm_blockwise without the workspace.
 *   When the automatically chosen variant's split-K scratch
 *   (fp8q_workspace_bytes(M, N, K, 1)) exceeds FP8Q_NOALLOC_SCRATCH_BYTES,
 *   the call runs that variant's tile shape with whole-K tiles (no scratch)
 *   instead.  A variant set by fp8q_force_gemm_variant is not changed: if its
 *   scratch does not fit, the call returns FP8Q_ERR_UNSUPPORTED and launches
 *   nothing.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   Every call clears the part of the array that must start at zero (the
 *   split-K arrival counters) with cudaMemsetAsync on its stream.
 *   All calls on a device share the one array: calls that can overlap on the
 *   GPU (different streams without ordering) race and give wrong results.
 */
#define FP8Q_NOALLOC_SCRATCH_BYTES (16u << 20)
FP8Q_API fp8q_status fp8q_scaled_mm_blockwise_noalloc(const void* a_q, const void* b_q,
                                                      const float* a_scale, int64_t as_stride_m,
                                                      int64_t as_stride_kb, const float* b_scale,
                                                      int64_t M, int64_t N, int64_t K, void* y,
                                                      int64_t ldy, void* stream);

/* ------------------------------------------------------------------------ */
/* W8A8_INT8                                                                 */
/* ------------------------------------------------------------------------ */

/*
 * The W8A8_INT8 scheme ("Helion linear backend" (aihirek.info), section
 * "Autotuning selects the variant": FP8_Dynamic, W8A8_INT8 and Block_FP8).
 * The pages name the scheme only; this library reads it as the FP8 path with
 * signed 8-bit integer codes:
 *   scale  s = fl32(max(amax, 1e-10) / 127)   (IEEE fp32 division)
 *   codes  q = int8(round-half-even(fl32(y / s))), saturated to [-128, 127]
 *   GEMM   y[m, n] = bf16_rn( sa(m) sb(n) sum_k qa[m,k] qb[n,k] ), the sum
 *          exact in 32-bit integers (tcgen05 kind::i8), converted to fp32
 * The quant entry points take the arguments of their FP8 counterparts (no
 * ue8m0); q holds int8 codes.  fp8q_scaled_mm_i8 takes those of
 * fp8q_scaled_mm (int8 operands; K <= 133152 keeps every integer sum in
 * range) with fp8q_workspace_bytes(M, N, K, 3).
 */
FP8Q_API fp8q_status fp8q_group_quant_i8(const void* x, int64_t M, int64_t K, int64_t ldx,
                                         int group_size, void* q, int64_t ldq, float* scales,
                                         int64_t s_stride_m, int64_t s_stride_g, void* stream);
FP8Q_API fp8q_status fp8q_rmsnorm_quant_i8(const void* x, const void* w, float eps, int64_t M,
                                           int64_t H, int64_t ldx, int group_size, void* q,
                                           int64_t ldq, float* scales, int64_t s_stride_m,
                                           int64_t s_stride_g, void* stream);
FP8Q_API fp8q_status fp8q_silu_mul_quant_i8(const void* x, int64_t M, int64_t I, int64_t ldx,
                                            int group_size, void* q, int64_t ldq, float* scales,
                                            int64_t s_stride_m, int64_t s_stride_g, void* stream);
FP8Q_API fp8q_status fp8q_scaled_mm_i8(const void* a_q, const void* b_q, const float* a_scale,
                                       int a_per_token, const float* b_scale, int b_per_channel,
                                       int64_t M, int64_t N, int64_t K, void* y, int64_t ldy,
                                       void* workspace, size_t ws_bytes, void* stream);

/* Bytes of scratch the GEMM of this shape needs (0 if none); blockwise = 0
 * (fp8q_scaled_mm), 1 (fp8q_scaled_mm_blockwise), 2
 * (fp8q_scaled_mm_blockwise_e8m0), 3 (fp8q_scaled_mm_i8).  Depends only on the shape and the variant
 * the library picks for it. */
FP8Q_API size_t fp8q_workspace_bytes(int64_t M, int64_t N, int64_t K, int blockwise);

/* ------------------------------------------------------------------------ */
/* GEMM variant selection (Split-K / Swap-AB / tile width)                   */
/* ------------------------------------------------------------------------ */

/* A GEMM variant ("Helion linear backend" (aihirek.info), section "Single
 * GEMM implementation handles several algorithms"): swap_ab = 1 computes
 * (B A^T)^T so the tokens sit in the MMA's N slot; split_k > 1 divides the K
 * loop of every output tile among that many CTAs; split_k = 0 selects
 * stream-K: every CTA (at most one per SM) takes an equal contiguous range of
 * (tile, K block) iterations and tiles cut by range boundaries are summed
 * from their pieces in a fixed order; block_n is the MMA N extent;
 * cta_pair = 1 runs each 256-row tile on a cluster of two CTAs (two SMs)
 * sharing one tcgen05 .cta_group::2 MMA, each SM staging half of the B tile
 * (only with swap_ab = 0 and split_k = 1; block_n 128, or 256 for the
 * per-token scheme).  block_n 224 (and 256 with one accumulator buffer) are
 * the E8M0 GEMM's wide tiles (no swap). */
typedef struct {
    int swap_ab;
    int split_k;
    int block_n;
    int cta_pair;
} fp8q_gemm_variant;

/* The variant the library would run for this shape: the row of its built-in
 * table of variants measured fastest on a B200 (the shapes of the Qwen3-8B
 * and Qwen3-32B linear layers, per bucket of M; written by the package's
 * tune.py), else a rule drawn from the same measurements.  The split_k it
 * reports is the one that runs (a split larger than the number of K blocks
 * is reduced).  Returns FP8Q_OK. */
FP8Q_API fp8q_status fp8q_select_gemm_variant(int64_t M, int64_t N, int64_t K, int blockwise,
                                     fp8q_gemm_variant* out);

/* Force a variant for every following GEMM call in this process (testing and
 * tuning only; not thread-safe).  NULL restores automatic selection.  Returns
 * FP8Q_ERR_INVALID_ARG if the variant is malformed (block_n not one of
 * 8, 16, 32, 64, 128, 224, 256; split_k < 0 or > 64; cta_pair not 0 or 1, or
 * set with another combination than the one above).  A GEMM call whose
 * scheme cannot run the forced variant returns FP8Q_ERR_UNSUPPORTED.
 * {swap_ab 1, split_k 1, block_n 8, cta_pair 0} is the decode variant: the
 * weights streamed through the warp-level MMA (mma.sync m16n8k32 e4m3) for
 * M <= 8 tokens, K a multiple of 128, per-token/per-channel or blockwise fp32
 * scales; no workspace. */
FP8Q_API fp8q_status fp8q_force_gemm_variant(const fp8q_gemm_variant* v);

/* ------------------------------------------------------------------------ */
/* Status                                                                    */
/* ------------------------------------------------------------------------ */

/* Synchronizes `stream`, then returns and clears the device status word of
 * the current device (FP8Q_OK; FP8Q_ERR_TIMEOUT if a kernel gave up on a
 * wait since the last read; FP8Q_ERR_INVALID_ARG if fp8q_qk_norm_rope met a
 * position outside its cache; the first error recorded wins).  FP8Q_ERR_CUDA
 * if the synchronization failed. */
FP8Q_API fp8q_status fp8q_last_device_status(void* stream);

/* Static description of a status code (never NULL). */
FP8Q_API const char* fp8q_status_string(fp8q_status s);

/* Library version string, e.g. "fp8q 0.1 sm_100a". */
FP8Q_API const char* fp8q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
