/*
 * fp8q_oracle.c -- plain, slow, obviously correct CPU oracle of the FP8 W8A8
 * linear path (dynamic activation quantization + scaled FP8 GEMM).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  Only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant generator
 * with the CUDA path.
 *
 * Source of what is computed.  The pages name the ops ("Helion in vLLM"
 * (24-ai.news), section "Kernels integrated into vLLM", items 1-3 and 5-9) but
 * never write out their arithmetic.  The arithmetic is fixed as:
 *   scale  s = fl32(max(amax, 1e-10) / 448)          (IEEE fp32 division)
 *   UE8M0  s <- smallest power of two >= s             (optional mode)
 *   code   q = e4m3fn(fl32(x / s)), round to nearest even, saturating at +-448
 *   groups contiguous 1x128 chunks of a row, or the whole row (per token)
 *   GEMM   y = bf16(sum_k (qa*sa)(qb*sb)), fp32 scales, bf16 output
 * Readings where nothing fixes a step:
 *   - RMSNorm: r = 1/sqrt(mean(x^2) + eps) in fp64; n = bf16(x*r); y = bf16(n*w).
 *   - SiLU*mul: gate = first half of the row, up = second half;
 *     y = bf16(silu(gate)*up), one rounding of the fp64 value.
 *   - the sign of zero is kept by the encoder (-tiny -> 0x80); NaN -> 0x7F.
 *
 * Floating point is fp64 except where the definition itself fixes fp32 (the
 * scale and the x/s division, whose result decides an integer code).
 * Rows are parallel under OpenMP; nothing else is blocked, fused or reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Number formats, written from their definitions.                           */
/* ------------------------------------------------------------------------ */

/* Round-half-to-even of a non-negative double to an integer-valued double. */
static double rne_integer(double n)
{
    double f = floor(n);
    double d = n - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* float8 e4m3fn: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * No infinities; 0x7F / 0xFF are NaN; largest finite 0x7E = 1.75 * 2^8 = 448.
 * Normals 2^-6 .. 448; subnormals k * 2^-9, k = 1..7. */
uint8_t oracle_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;          /* saturate */
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);                               /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                              /* floor(log2 a) */
    if (E < -6) E = -6;                          /* subnormal binade shares 2^-6's quantum */
    double quantum = ldexp(1.0, E - 3);          /* 3 mantissa bits */
    double r = rne_integer(a / quantum);         /* a / quantum is exact */
    double val = r * quantum;                    /* <= 448 because a < 448 */
    if (val == 0.0) return sign;
    if (val < ldexp(1.0, -6)) {                  /* subnormal: val = k * 2^-9 */
        return sign | (uint8_t)(val / ldexp(1.0, -9));
    }
    frexp(val, &e2);
    int Ev = e2 - 1;
    int mant = (int)(val / ldexp(1.0, Ev) * 8.0) - 8;   /* 0..7 */
    return sign | (uint8_t)(((Ev + 7) << 3) | mant);
}

/* Value of an e4m3fn code (NaN codes give NaN). */
double oracle_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
static double bf16_bits_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bfloat16 (8 significant bits, binary32
 * exponent range: min normal 2^-126, subnormal quantum 2^-133), ties to even.
 * Returns the rounded value as a float (always exactly representable). */
float oracle_bf16_round(double v)
{
    if (isnan(v)) return (float)v;
    double a = fabs(v);
    if (a == 0.0) return (float)v;
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;
    if (E < -126) E = -126;
    double quantum = ldexp(1.0, E - 7);
    double r = rne_integer(a / quantum) * quantum;
    if (r >= ldexp(2.0, 127)) r = INFINITY;      /* beyond the largest finite bf16 */
    return (float)(v < 0 ? -r : r);
}

/* The dynamic scale of a group whose largest magnitude is amax. */
float oracle_scale(float amax, int ue8m0)
{
    float s = fmaxf(amax, 1e-10f) / 448.0f;      /* IEEE fp32 division */
    if (ue8m0) {
        int e2;
        float f = frexpf(s, &e2);                /* s = f * 2^e2, f in [0.5, 1) */
        if (f != 0.5f) s = ldexpf(1.0f, e2);     /* round up to the next power of two */
    }
    return s;
}

/* E8M0 ("UE8M0"): an 8-bit unsigned biased exponent, bias 127, no sign and no
 * mantissa; byte b stands for 2^(b - 127); b = 255 is NaN.  It is the packed
 * storage of a power-of-two scale: the exponent byte that the FP8 GEMM pages'
 * B200 path needs ("Helion in vLLM", section "Practical limits": UE8M0 scales
 * for DeepGEMM on B200).  Encode takes a scale that must be a power of two
 * in [2^-127, 2^127] and returns its byte; anything else gives 255. */
uint8_t oracle_e8m0_encode(float s)
{
    if (!(s > 0.0f) || isinf(s)) return 0xFF;
    int e2;
    double f = frexp((double)s, &e2);            /* s = f * 2^e2, f in [0.5, 1) */
    if (f != 0.5) return 0xFF;                   /* not a power of two */
    int e = e2 - 1;                              /* s = 2^e */
    if (e < -127 || e > 127) return 0xFF;
    return (uint8_t)(e + 127);
}

double oracle_e8m0_decode(uint8_t b)
{
    if (b == 0xFF) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* Quantize L values of one group: scale from the group's amax, then codes. */
static void quantize_group(const float* v, int64_t L, int ue8m0, uint8_t* q, float* s_out)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < L; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    float s = oracle_scale(amax, ue8m0);
    for (int64_t i = 0; i < L; ++i) q[i] = oracle_e4m3_encode(v[i] / s);
    *s_out = s;
}

/* Quantize one row of length K in groups of g (g == K: per token).
 * Scales go to s[0 .. K/g). */
static void quantize_row(const float* y, int64_t K, int64_t g, int ue8m0, uint8_t* q, float* s)
{
    for (int64_t j = 0; j < K / g; ++j) quantize_group(y + j * g, g, ue8m0, q + j * g, s + j);
}

/* ------------------------------------------------------------------------ */
/* Activation quantization ops.  Outputs: q [M, K] row-major (ld = K),       */
/* s [M, K/g] row-major, optional y [M, K] (the values that were quantized). */
/* ------------------------------------------------------------------------ */

/* per_token_group_fp8_quant / dynamic_per_token_scaled_fp8_quant
 * ("Helion in vLLM", "Kernels integrated into vLLM", items 5 and 1). */
void oracle_group_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int64_t g,
                        int ue8m0, uint8_t* q, float* s, float* y_out)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        float* y = (float*)malloc(sizeof(float) * (size_t)K);
        for (int64_t k = 0; k < K; ++k) y[k] = (float)bf16_bits_value(x[m * ldx + k]);
        quantize_row(y, K, g, ue8m0, q + m * K, s + m * (K / g));
        if (y_out) memcpy(y_out + m * K, y, sizeof(float) * (size_t)K);
        free(y);
    }
}

/* rms_norm_dynamic_per_token_quant (g == H) and rms_norm_per_block_quant
 * (g == 128) ("Helion in vLLM", "Kernels integrated into vLLM", items 2, 6).
 * The norm is taken over the whole row; the scales per group. */
void oracle_rmsnorm_quant(const uint16_t* x, const uint16_t* w, float eps, int64_t M, int64_t H,
                          int64_t ldx, int64_t g, int ue8m0, uint8_t* q, float* s, float* y_out)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* xr = x + m * ldx;
        double sumsq = 0.0;
        for (int64_t k = 0; k < H; ++k) {
            double v = bf16_bits_value(xr[k]);
            sumsq += v * v;
        }
        double r = 1.0 / sqrt(sumsq / (double)H + (double)eps);
        float* y = (float*)malloc(sizeof(float) * (size_t)H);
        for (int64_t k = 0; k < H; ++k) {
            double n = oracle_bf16_round(bf16_bits_value(xr[k]) * r);
            y[k] = oracle_bf16_round(n * bf16_bits_value(w[k]));
        }
        quantize_row(y, H, g, ue8m0, q + m * H, s + m * (H / g));
        if (y_out) memcpy(y_out + m * H, y, sizeof(float) * (size_t)H);
        free(y);
    }
}

/* Residual-add variant of the RMSNorm quant (the fusion "on either side of
 * the path" that continues the pages' call-count reduction, "Helion in vLLM",
 * section "Kernels integrated into vLLM").  Reading: the fused op feeds the
 * norm what the unfused chain would -- the residual stream is kept in the
 * model dtype, so h = bf16(x + residual) with one rounding of the exact sum;
 * h is written to res_out and then RMSNorm-quantized exactly as
 * oracle_rmsnorm_quant does. */
void oracle_add_rmsnorm_quant(const uint16_t* x, const uint16_t* res, const uint16_t* w, float eps,
                              int64_t M, int64_t H, int64_t g, int ue8m0, uint8_t* q, float* s,
                              uint16_t* res_out, float* y_out)
{
    uint16_t* h = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(M * H));
    for (int64_t i = 0; i < M * H; ++i) {
        float v = oracle_bf16_round(bf16_bits_value(x[i]) + bf16_bits_value(res[i]));
        uint32_t u;
        memcpy(&u, &v, 4);
        h[i] = (uint16_t)(u >> 16);              /* v is a bf16 value: its upper half */
    }
    oracle_rmsnorm_quant(h, w, eps, M, H, H, g, ue8m0, q, s, y_out);
    memcpy(res_out, h, sizeof(uint16_t) * (size_t)(M * H));
    free(h);
}

/* silu_and_mul_dynamic_per_token_quant (g == I) and silu_and_mul_per_block_quant
 * (g == 128) ("Helion in vLLM", "Kernels integrated into vLLM", items 3, 7).
 * Input row [gate(I) | up(I)]; silu(t) = t / (1 + e^-t). */
void oracle_silu_mul_quant(const uint16_t* x, int64_t M, int64_t I, int64_t ldx, int64_t g,
                           int ue8m0, uint8_t* q, float* s, float* y_out)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* xr = x + m * ldx;
        float* y = (float*)malloc(sizeof(float) * (size_t)I);
        for (int64_t k = 0; k < I; ++k) {
            double gt = bf16_bits_value(xr[k]);
            double up = bf16_bits_value(xr[I + k]);
            double silu = gt / (1.0 + exp(-gt));
            y[k] = oracle_bf16_round(silu * up);
        }
        quantize_row(y, I, g, ue8m0, q + m * I, s + m * (I / g));
        if (y_out) memcpy(y_out + m * I, y, sizeof(float) * (size_t)I);
        free(y);
    }
}

/* ------------------------------------------------------------------------ */
/* Scaled FP8 GEMMs.  y_ref[m, n] = sum_k (Ea[m,k] sa)(Eb[n,k] sb) in fp64,   */
/* absdot[m, n] = sum_k |(Ea sa)(Eb sb)|.  A is [M, K], B is [N, K] (both     */
/* K-contiguous, as nn.Linear stores weights); only the listed rows of A are  */
/* computed, into row i of the outputs for rows[i].                          */
/* ------------------------------------------------------------------------ */

static double g_dec[256];
static int g_dec_ready = 0;

static void dec_table_init(void)
{
    if (g_dec_ready) return;
    for (int c = 0; c < 256; ++c) g_dec[c] = oracle_e4m3_decode((uint8_t)c);
    g_dec_ready = 1;
}

/* scaled_mm ("Helion in vLLM", "Kernels integrated into vLLM", item 8):
 * per-token (sa[M]) or per-tensor (sa[0]) activation scales, per-channel
 * (sb[N]) or per-tensor (sb[0]) weight scales. */
void oracle_scaled_mm_rows(const uint8_t* a, const uint8_t* b, const float* sa, int a_per_token,
                           const float* sb, int b_per_channel, int64_t M, int64_t N, int64_t K,
                           const int64_t* rows, int64_t nrows, double* y, double* absdot)
{
    (void)M;
    dec_table_init();
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows[i];
            double s_a = a_per_token ? sa[m] : sa[0];
            double s_b = b_per_channel ? sb[n] : sb[0];
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double t = (g_dec[a[m * K + k]] * s_a) * (g_dec[b[n * K + k]] * s_b);
                acc += t;
                aacc += fabs(t);
            }
            y[i * N + n] = acc;
            absdot[i * N + n] = aacc;
        }
    }
}

/* scaled_mm_blockwise ("Helion in vLLM", "Kernels integrated into vLLM",
 * item 9; the Block_FP8 scheme of "Helion linear backend" (aihirek.info),
 * section "Autotuning selects the variant"): sa [M, K/128] row-major, one
 * scale per 1x128 activation group; sb [N/128, K/128] row-major, one scale
 * per 128x128 weight block. */
void oracle_scaled_mm_blockwise_rows(const uint8_t* a, const uint8_t* b, const float* sa,
                                     const float* sb, int64_t M, int64_t N, int64_t K,
                                     const int64_t* rows, int64_t nrows, double* y, double* absdot)
{
    (void)M;
    dec_table_init();
    const int64_t KB = K / 128;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows[i];
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double s_a = sa[m * KB + k / 128];
                double s_b = sb[(n / 128) * KB + k / 128];
                double t = (g_dec[a[m * K + k]] * s_a) * (g_dec[b[n * K + k]] * s_b);
                acc += t;
                aacc += fabs(t);
            }
            y[i * N + n] = acc;
            absdot[i * N + n] = aacc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Array helpers for the pins (plain loops over the scalar definitions).     */
/* ------------------------------------------------------------------------ */

void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_decode_array(const uint8_t* c, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

void oracle_bf16_round_array(const double* v, int64_t n, float* out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_round(v[i]);
}

void oracle_scale_array(const float* amax, int64_t n, int ue8m0, float* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_scale(amax[i], ue8m0);
}

void oracle_e8m0_encode_array(const float* s, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e8m0_encode(s[i]);
}

void oracle_e8m0_decode_array(const uint8_t* b, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e8m0_decode(b[i]);
}

/* ------------------------------------------------------------------------ */
/* W8A8_INT8 ("Helion linear backend" (aihirek.info), section "Autotuning    */
/* selects the variant": the W8A8_INT8 scheme next to FP8_Dynamic and        */
/* Block_FP8).  The pages name the scheme only; the reading taken is the     */
/* FP8 path's with int8 codes:                                               */
/*   scale s = fl32(max(amax, 1e-10) / 127)      (IEEE fp32 division)         */
/*   code  q = int8(RNE(fl32(y / s))), saturated to [-128, 127]              */
/*   GEMM  y = bf16(sa * sb * sum_k qa * qb), the sum exact in integers.     */
/* ------------------------------------------------------------------------ */

/* Nearest integer (ties to even) of an fp32 value, saturated to int8; NaN -> 0. */
int8_t oracle_int8_encode(float v)
{
    if (isnan(v)) return 0;
    double a = fabs((double)v);
    double r = rne_integer(a);
    if (v < 0) r = -r;
    if (r > 127.0) r = 127.0;
    if (r < -128.0) r = -128.0;
    return (int8_t)r;
}

float oracle_int8_scale(float amax)
{
    return fmaxf(amax, 1e-10f) / 127.0f;         /* IEEE fp32 division */
}

/* Quantize M rows of L values (the values a producer op feeds the quantizer)
 * in groups of g to int8 codes, scales s [M, L/g] row-major. */
void oracle_int8_quant_rows(const float* y, int64_t M, int64_t L, int64_t g, int8_t* q, float* s)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t j = 0; j < L / g; ++j) {
            const float* v = y + m * L + j * g;
            float amax = 0.0f;
            for (int64_t i = 0; i < g; ++i) {
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            float sc = oracle_int8_scale(amax);
            for (int64_t i = 0; i < g; ++i) q[m * L + j * g + i] = oracle_int8_encode(v[i] / sc);
            s[m * (L / g) + j] = sc;
        }
    }
}

/* int8 scaled_mm: y_ref[m, n] = sa * sb * sum_k qa[m,k] qb[n,k] (the integer
 * sum exact in int64), absdot = |sa sb| sum_k |qa qb|. */
void oracle_scaled_mm_i8_rows(const int8_t* a, const int8_t* b, const float* sa, int a_per_token,
                              const float* sb, int b_per_channel, int64_t M, int64_t N, int64_t K,
                              const int64_t* rows, int64_t nrows, double* y, double* absdot)
{
    (void)M;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows[i];
            int64_t acc = 0, aacc = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t t = (int64_t)a[m * K + k] * (int64_t)b[n * K + k];
                acc += t;
                aacc += t < 0 ? -t : t;
            }
            double sc = (double)(a_per_token ? sa[m] : sa[0]) * (double)(b_per_channel ? sb[n] : sb[0]);
            y[i * N + n] = (double)acc * sc;
            absdot[i * N + n] = (double)aacc * fabs(sc);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* fused_qk_norm_rope (vllm PR #44010 page, section "Code analysis": the op  */
/* takes qkv, the q / k / v head counts, head_dim, eps, q_weight, k_weight,  */
/* the rope cos_sin_cache, is_neox and positions; "Helion in vLLM", section  */
/* "Kernels integrated into vLLM", item 4).  Reading taken (the pages print  */
/* no arithmetic):                                                           */
/*   qkv row t = [q heads (hq) | k heads (hk) | v heads (hv)], D each, bf16; */
/*   every q and k head: the RMSNorm of this library over its D values       */
/*     r = 1/sqrt(mean(x^2) + eps), n = bf16(x r), y = bf16(n w)             */
/*   (w = q_weight or k_weight, [D]), then the rotary embedding at position  */
/*   p = positions[t] with cos = cache[p][0 .. D/2), sin = cache[p][D/2 .. D) */
/*   (fp32 cache), pairs (i, i + D/2) when is_neox, else (2i, 2i + 1):       */
/*     out_a = bf16(y_a cos_i - y_b sin_i),  out_b = bf16(y_b cos_i + y_a sin_i) */
/*   written back in place; v heads are left as they are.                    */
/* ------------------------------------------------------------------------ */
void oracle_qk_norm_rope(uint16_t* qkv, int64_t T, int64_t ld, int64_t hq, int64_t hk, int64_t D,
                         float eps, const uint16_t* qw, const uint16_t* kw, const float* cos_sin,
                         const int64_t* positions, int is_neox)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double* y = (double*)malloc(sizeof(double) * (size_t)D);
        const float* cs = cos_sin + positions[t] * D;
        for (int64_t h = 0; h < hq + hk; ++h) {
            uint16_t* x = qkv + t * ld + h * D;
            const uint16_t* w = h < hq ? qw : kw;
            double ss = 0.0;
            for (int64_t i = 0; i < D; ++i) {
                double v = bf16_bits_value(x[i]);
                ss += v * v;
            }
            double r = 1.0 / sqrt(ss / (double)D + (double)eps);
            for (int64_t i = 0; i < D; ++i) {
                double n = oracle_bf16_round(bf16_bits_value(x[i]) * r);
                y[i] = oracle_bf16_round(n * bf16_bits_value(w[i]));
            }
            for (int64_t i = 0; i < D / 2; ++i) {
                int64_t a = is_neox ? i : 2 * i;
                int64_t b = is_neox ? i + D / 2 : 2 * i + 1;
                double c = cs[i], sn = cs[D / 2 + i];
                float oa = oracle_bf16_round(y[a] * c - y[b] * sn);
                float ob = oracle_bf16_round(y[b] * c + y[a] * sn);
                uint32_t ua, ub;
                memcpy(&ua, &oa, 4);
                memcpy(&ub, &ob, 4);
                x[a] = (uint16_t)(ua >> 16);
                x[b] = (uint16_t)(ub >> 16);
            }
        }
        free(y);
    }
}
