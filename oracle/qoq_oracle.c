/*
 * qoq_oracle.c -- plain, slow CPU oracle for the QoQ W4A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent definition that the
 * CUDA library is checked against.  Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it; the product path never does.
 * It shares no code, header, table or constant generator with the CUDA
 * library, and it includes nothing from it.
 *
 * Every function below follows one passage of the pages, cited by page title
 * and section/equation:
 *
 *   [LBW]   "QServe: Low Bit Width Does Not Guarantee High Throughput"
 *           (and its Chinese twin "QServe：低比特不等于高吞吐"),
 *           section 4 "Formalization and procedure": the stage-1 equation
 *           (per-channel symmetric INT8 in the protective range [-119,119])
 *           and the stage-2 equation (group-wise asymmetric UINT4 in the INT8
 *           domain), plus the paragraph after them (multiply by the integer
 *           scale first, then subtract the precomputed zero compensation).
 *   [CARD]  "QServe: W4A8KV4 Quantization and System Co-design for Efficient
 *           LLM Serving" (paper card), "Key points", progressive group
 *           quantization bullets: per-channel FP16 scales, protective range.
 *   [GUIDE] "QServe Guide: W4A8KV4 Quantization for LLM Serving",
 *           "Deep Dive: Mathematical Formulation and Hardware Alignment",
 *           subsection 1 "Per-Channel Weight and Per-Token Activation Scaling
 *           Mechanics": the per-token activation equation and the output
 *           rescaling equation; and "The Architecture", subsection 2
 *           "High-Throughput Native INT8 Tensor Core GEMMs": INT32
 *           accumulation, scales applied once after the inner product.
 *
 * Readings of points the pages leave open:
 *   - "round" is round-half-to-even (IEEE rint in the default mode).
 *   - s_c and s_x are stored as FP16 (round to nearest even) and the stored,
 *     rounded value is the one used to quantize.
 *   - A zero scale (all-zero row, or a scale that rounds to FP16 zero) gives
 *     an all-zero quantized row; no division happens.
 *   - Stage 2 (the pages give q and W-hat but not how s_g and z are chosen):
 *       mn = min(0, min W8), mx = max(0, max W8) over the group,
 *       s_g = max(1, ceil((mx - mn) / 15))  (integer),
 *       z   = round_half_even(-mn / s_g)    (exact rational rounding),
 *       q   = clamp(round_half_even(W8 / s_g) + z, 0, 15),
 *       zs  = z * s_g  (the precomputed zero compensation).
 *   - Epilogue order: Y = fp16_rn( ((float)acc * sx) * sc ) in FP32.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -fopenmp -ffp-contract=off
 * (no fast-math: every float operation is a single IEEE-rounded step).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 <-> binary32, written from the format definition.       */
/* ------------------------------------------------------------------------ */

/* Exact widening of a binary16 bit pattern to binary32. */
float oracle_half_to_float(uint16_t h)
{
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t expo = (h >> 10) & 0x1fu;
    uint32_t mant = h & 0x3ffu;
    uint32_t bits;
    if (expo == 0x1fu) {                         /* inf / nan */
        bits = sign | 0x7f800000u | (mant << 13);
    } else if (expo != 0) {                      /* normal */
        bits = sign | ((expo - 15u + 127u) << 23) | (mant << 13);
    } else {                                     /* zero / subnormal: mant * 2^-24 */
        float v = (float)mant * 5.9604644775390625e-08f;   /* 2^-24, exact */
        memcpy(&bits, &v, 4);
        bits |= sign;
    }
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

/* binary32 -> binary16, round to nearest, ties to even. */
uint16_t oracle_float_to_half_rn(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;

    if (ax > 0x7f800000u)                        /* nan: keep it a quiet nan */
        return (uint16_t)(sign | 0x7e00u);
    if (ax >= 0x477ff000u)                       /* >= 65520 rounds to inf */
        return (uint16_t)(sign | 0x7c00u);
    if (ax < 0x38800000u) {                      /* below 2^-14: subnormal half */
        float a;
        memcpy(&a, &ax, 4);
        /* |f| * 2^24 is exact (power-of-two scaling of a value < 2^-14);
         * rintf rounds to the nearest integer count of 2^-24, ties to even. */
        float units = rintf(a * 16777216.0f);
        return (uint16_t)(sign | (uint16_t)units);   /* 1024 -> 0x0400, the min normal */
    }
    /* normal range: keep 10 of the 23 mantissa bits, round the other 13 */
    uint32_t expo = (ax >> 23) - 127u + 15u;
    uint32_t mant = ax & 0x7fffffu;
    uint32_t h = (expo << 10) | (mant >> 13);
    uint32_t rem = mant & 0x1fffu;
    if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
        h += 1u;                                 /* a carry into the exponent is correct */
    return (uint16_t)(sign | h);
}

/* ------------------------------------------------------------------------ */
/* Integer helper: round_half_even(a / b) for b > 0, exact.                  */
/* ------------------------------------------------------------------------ */
int oracle_div_round_half_even(int a, int b)
{
    int f = a / b;                 /* C truncates toward zero; make it floor */
    int r = a - f * b;
    if (r < 0) { f -= 1; r += b; } /* now a = f*b + r with 0 <= r < b */
    if (2 * r > b) return f + 1;
    if (2 * r < b) return f;
    return (f % 2 == 0) ? f : f + 1;
}

/* ------------------------------------------------------------------------ */
/* Stage 2 for one group: [LBW] section 4, stage-2 equation.                 */
/* ------------------------------------------------------------------------ */
void oracle_stage2_group(const int8_t *W8, int G,
                         uint8_t *q, uint8_t *s_g, uint8_t *z, uint8_t *zs)
{
    int mn = 0, mx = 0;
    for (int i = 0; i < G; ++i) {
        if (W8[i] < mn) mn = W8[i];
        if (W8[i] > mx) mx = W8[i];
    }
    int range = mx - mn;
    int sg = (range + 14) / 15;            /* ceil(range / 15) */
    if (sg < 1) sg = 1;
    int zz = oracle_div_round_half_even(-mn, sg);
    for (int i = 0; i < G; ++i) {
        int v = oracle_div_round_half_even(W8[i], sg) + zz;
        if (v < 0) v = 0;
        if (v > 15) v = 15;
        q[i] = (uint8_t)v;
    }
    *s_g = (uint8_t)sg;
    *z = (uint8_t)zz;
    *zs = (uint8_t)(zz * sg);
}

/* ------------------------------------------------------------------------ */
/* Stages 1 + 2 for a weight matrix W [N][K] (row n = output channel).       */
/* Stage 1: [LBW] section 4, stage-1 equation; FP16 scale per [CARD].        */
/* Outputs are canonical row-major arrays:                                   */
/*   s_c [N] (FP16 bits), W8 [N][K], q [N][K] (0..15, one per byte),        */
/*   s_g, z, zs [N][K/G].                                                    */
/* ------------------------------------------------------------------------ */
void oracle_quantize_weights(const float *W, int64_t N, int64_t K, int64_t G,
                             uint16_t *s_c, int8_t *W8, uint8_t *q,
                             uint8_t *s_g, uint8_t *z, uint8_t *zs)
{
    int64_t ng = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const float *w = W + n * K;
        int8_t *w8 = W8 + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(w[k]);
            if (a > amax) amax = a;
        }
        uint16_t sc_bits = oracle_float_to_half_rn(amax / 119.0f);
        float sc = oracle_half_to_float(sc_bits);
        s_c[n] = sc_bits;
        for (int64_t k = 0; k < K; ++k) {
            if (sc == 0.0f) { w8[k] = 0; continue; }
            float r = rintf(w[k] / sc);
            if (r > 119.0f) r = 119.0f;
            if (r < -119.0f) r = -119.0f;
            w8[k] = (int8_t)r;
        }
        for (int64_t g = 0; g < ng; ++g)
            oracle_stage2_group(w8 + g * G, (int)G, q + n * K + g * G,
                                s_g + n * ng + g, z + n * ng + g, zs + n * ng + g);
    }
}

/* ------------------------------------------------------------------------ */
/* INT4 -> INT8: multiply by the integer group scale, then subtract the      */
/* precomputed zero compensation ([LBW] section 4, paragraph after the       */
/* stage-2 equation; [CARD] "multiplies first and subtracts afterward").     */
/* ------------------------------------------------------------------------ */
void oracle_dequant_weights(const uint8_t *q, const uint8_t *s_g, const uint8_t *zs,
                            int64_t N, int64_t K, int64_t G, int8_t *W8hat)
{
    int64_t ng = K / G;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = k / G;
            int v = (int)q[n * K + k] * (int)s_g[n * ng + g] - (int)zs[n * ng + g];
            W8hat[n * K + k] = (int8_t)v;   /* in [-127,127] for quantizer output */
        }
}

/* ------------------------------------------------------------------------ */
/* Per-token symmetric INT8 activations: [GUIDE] subsection 1, activation    */
/* equation (Delta_x = max|X| / 127, clamp(round(X / Delta_x), -128, 127)).   */
/* X [M][K] FP16 bits -> X8 [M][K], s_x [M] FP16 bits.                      */
/* ------------------------------------------------------------------------ */
void oracle_quant_act(const uint16_t *X, int64_t M, int64_t K,
                      int8_t *X8, uint16_t *s_x)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t *x = X + m * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(oracle_half_to_float(x[k]));
            if (a > amax) amax = a;
        }
        uint16_t sx_bits = oracle_float_to_half_rn(amax / 127.0f);
        float sx = oracle_half_to_float(sx_bits);
        s_x[m] = sx_bits;
        for (int64_t k = 0; k < K; ++k) {
            if (sx == 0.0f) { X8[m * K + k] = 0; continue; }
            float r = rintf(oracle_half_to_float(x[k]) / sx);
            if (r > 127.0f) r = 127.0f;
            if (r < -128.0f) r = -128.0f;
            X8[m * K + k] = (int8_t)r;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* INT32 inner products: [GUIDE] "The Architecture" subsection 2 (INT8 x     */
/* INT8 products accumulated in INT32).  acc[m][n] = sum_k X8[m][k]*W8hat[n][k]. */
/* Accumulated in int64 and narrowed; |acc| <= K*128*127 < 2^31 for          */
/* K <= 132104, which the caller guarantees.                                 */
/* ------------------------------------------------------------------------ */
void oracle_gemm_i32(const int8_t *X8, const int8_t *W8hat,
                     int64_t M, int64_t N, int64_t K, int32_t *acc)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            const int8_t *x = X8 + m * K;
            const int8_t *w = W8hat + n * K;
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)x[k] * (int64_t)w[k];
            acc[m * N + n] = (int32_t)s;
        }
}

/* ------------------------------------------------------------------------ */
/* Epilogue: [GUIDE] subsection 1, output rescaling equation: the per-token  */
/* and per-channel scales multiply the INT32 sum once, after the K loop.     */
/* Y[m][n] = fp16_rn( ((float)acc * sx[m]) * sc[n] ).                        */
/* ------------------------------------------------------------------------ */
void oracle_epilogue(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c,
                     int64_t M, int64_t N, uint16_t *Y)
{
    for (int64_t m = 0; m < M; ++m) {
        float sx = oracle_half_to_float(s_x[m]);
        for (int64_t n = 0; n < N; ++n) {
            float sc = oracle_half_to_float(s_c[n]);
            float a = (float)acc[m * N + n];
            float t = a * sx;
            float y = t * sc;
            Y[m * N + n] = oracle_float_to_half_rn(y);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* The W8A8 yardstick's weights ("QServe: Low Bit Width Does Not Guarantee   */
/* High Throughput", section 2 "Motivation": W8A8 keeps 8-bit weights and    */
/* 8-bit activations on INT8 tensor cores; the same page's Figure 3 roofline */
/* compares it with W4A16 and W4A8).  Reading: per-channel symmetric INT8    */
/* over the full range, s_w = fp16(max|W_n| / 127), W8 = clamp(round(W /    */
/* s_w), -127, 127), round half to even, with the stored FP16 scale; a zero  */
/* scale gives a zero row.  The product and the epilogue are the W4A8        */
/* layer's (oracle_gemm_i32, oracle_epilogue) with W8 in place of W8hat.      */
/* ------------------------------------------------------------------------ */
void oracle_quantize_weights_w8(const float *W, int64_t N, int64_t K, uint16_t *s_w, int8_t *W8)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const float *w = W + n * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(w[k]);
            if (a > amax) amax = a;
        }
        uint16_t bits = oracle_float_to_half_rn(amax / 127.0f);
        float sw = oracle_half_to_float(bits);
        s_w[n] = bits;
        for (int64_t k = 0; k < K; ++k) {
            if (sw == 0.0f) { W8[n * K + k] = 0; continue; }
            float r = rintf(w[k] / sw);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            W8[n * K + k] = (int8_t)r;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* binary64 -> binary16, round to nearest, ties to even, from the format     */
/* definition (11 significant bits; subnormals in units of 2^-24).            */
/* ------------------------------------------------------------------------ */
uint16_t oracle_double_to_half_rn(double d)
{
    uint16_t sign = signbit(d) ? 0x8000u : 0u;
    double a = fabs(d);
    if (isnan(d)) return (uint16_t)(sign | 0x7e00u);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);       /* rounds to inf */
    if (a < 6.103515625e-05) {                                  /* below 2^-14: subnormal */
        double units = nearbyint(a * 16777216.0);               /* exact scaling, RN-even */
        return (uint16_t)(sign | (uint16_t)units);              /* 1024 -> min normal */
    }
    int ex = 0;
    (void)frexp(a, &ex);                                        /* a = f * 2^ex, f in [0.5, 1) */
    double q = nearbyint(ldexp(a, 11 - ex));                    /* 11 significant bits */
    if (q >= 2048.0) { q = 1024.0; ex += 1; }
    return (uint16_t)(sign | (uint16_t)(((ex + 14) << 10) | ((int)q - 1024)));
}

/* ------------------------------------------------------------------------ */
/* Output-side fusion (the steps after the layer; the pages name the layer's */
/* epilogue, [GUIDE] "The Architecture" subsection 2, but not what follows). */
/* Readings: the fused result equals the unfused sequence.                    */
/*                                                                            */
/* Residual add: the layer's FP16 output y (as oracle_epilogue), then        */
/*   Y[m][n] = fp16_rn( (float)y + (float)R[m][n] )   (an FP16 add).          */
/* ------------------------------------------------------------------------ */
void oracle_epilogue_residual(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c,
                              int64_t M, int64_t N, const uint16_t *R, uint16_t *Y)
{
    for (int64_t m = 0; m < M; ++m) {
        float sx = oracle_half_to_float(s_x[m]);
        for (int64_t n = 0; n < N; ++n) {
            float sc = oracle_half_to_float(s_c[n]);
            float t = (float)acc[m * N + n] * sx;
            uint16_t y = oracle_float_to_half_rn(t * sc);
            float sum = oracle_half_to_float(y) + oracle_half_to_float(R[m * N + n]);
            Y[m * N + n] = oracle_float_to_half_rn(sum);
        }
    }
}

/* SiLU-gated product of a gate/up pair (the MLP activation that follows a   */
/* fused gate/up projection).  acc has N2 = 2*I columns in their natural     */
/* order: gate channel j at column j, up channel j at column I + j.  With    */
/* g and u the layer's FP16 outputs of those two columns,                    */
/*   Out[m][j] = fp16_rn( g / (1 + exp(-g)) * u )   evaluated in binary64.  */
/* ------------------------------------------------------------------------ */
void oracle_epilogue_silu_mul(const int32_t *acc, const uint16_t *s_x, const uint16_t *s_c,
                              int64_t M, int64_t N2, uint16_t *Out)
{
    int64_t I = N2 / 2;
    for (int64_t m = 0; m < M; ++m) {
        float sx = oracle_half_to_float(s_x[m]);
        for (int64_t j = 0; j < I; ++j) {
            float tg = (float)acc[m * N2 + j] * sx;
            float tu = (float)acc[m * N2 + I + j] * sx;
            uint16_t g = oracle_float_to_half_rn(tg * oracle_half_to_float(s_c[j]));
            uint16_t u = oracle_float_to_half_rn(tu * oracle_half_to_float(s_c[I + j]));
            double gd = (double)oracle_half_to_float(g);
            double ud = (double)oracle_half_to_float(u);
            double silu = gd / (1.0 + exp(-gd));
            Out[m * I + j] = oracle_double_to_half_rn(silu * ud);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* KV4 decode attention with SmoothAttention.                                 */
/*                                                                            */
/* [LBW] section 4 (the SmoothAttention paragraph) and [GUIDE] "The           */
/* Architecture" subsection 3: a per-channel factor lambda_c moves the        */
/* outliers of the cached keys into the (uncached) query, K'_c = K_c /        */
/* lambda_c and Q'_c = Q_c * lambda_c, so Q'K'^T = QK^T; lambda_c =           */
/* max|K_c|^alpha, alpha = 0.5.  The smoothed keys and the values are stored */
/* as 4-bit integers with per-channel scales.  Readings where the pages are   */
/* silent:                                                                    */
/*   - the statistics are per (sequence, KV head, channel c), over the       */
/*     cached tokens; lambda is stored in FP16, floored at 1e-5 (a zero      */
/*     channel keeps a finite factor), computed as fp16(sqrt(max|K|)) for    */
/*     alpha = 0.5 and as fp16(pow(max|K|, alpha)) otherwise, in binary64;   */
/*   - K' = (float)K / (float)lambda in FP32 (IEEE division);                */
/*   - 4-bit codes are symmetric: s_c = fp16(max_l |X'[l][c]| / 7) in FP32,  */
/*     code = clamp(round(X' / s_c), -8, 7), round half to even; a zero      */
/*     scale gives zero codes (the same rule as the guide's illustration,    */
/*     applied per channel);                                                  */
/*   - attention for one new query token per sequence and query head h      */
/*     (KV head h / G, G = Hq / Hkv): score_l = sum_c Q'_c K^_lc / sqrt(d)    */
/*     with K^ = s_k * code, softmax over the L cached tokens, out_c =      */
/*     sum_l p_l V^_lc, all in binary64, output rounded once to FP16.        */
/* ------------------------------------------------------------------------ */
void oracle_smooth_lambda(const uint16_t *K, int64_t L, int64_t d, double alpha, uint16_t *lambda)
{
    for (int64_t c = 0; c < d; ++c) {
        float m = 0.0f;
        for (int64_t l = 0; l < L; ++l) {
            float a = fabsf(oracle_half_to_float(K[l * d + c]));
            if (a > m) m = a;
        }
        double v = (alpha == 0.5) ? sqrt((double)m) : pow((double)m, alpha);
        if (v < 1e-5) v = 1e-5;
        lambda[c] = oracle_double_to_half_rn(v);
    }
}

/* X [L][d] FP16 bits -> codes [L][d] (int8 in -8..7) and s [d] FP16 bits.
 * lambda (FP16 bits [d]) or NULL: the keys are divided by it first. */
void oracle_kv4_quantize(const uint16_t *X, int64_t L, int64_t d, const uint16_t *lambda,
                         int8_t *codes, uint16_t *s)
{
    for (int64_t c = 0; c < d; ++c) {
        float lam = lambda ? oracle_half_to_float(lambda[c]) : 1.0f;
        float m = 0.0f;
        for (int64_t l = 0; l < L; ++l) {
            float x = oracle_half_to_float(X[l * d + c]);
            if (lambda) x = x / lam;
            float a = fabsf(x);
            if (a > m) m = a;
        }
        uint16_t sb = oracle_float_to_half_rn(m / 7.0f);
        float sc = oracle_half_to_float(sb);
        s[c] = sb;
        for (int64_t l = 0; l < L; ++l) {
            float x = oracle_half_to_float(X[l * d + c]);
            if (lambda) x = x / lam;
            if (sc == 0.0f) { codes[l * d + c] = 0; continue; }
            float r = rintf(x / sc);
            if (r > 7.0f) r = 7.0f;
            if (r < -8.0f) r = -8.0f;
            codes[l * d + c] = (int8_t)r;
        }
    }
}

/* One sequence: q [Hq][d] FP16 bits (the unsmoothed query), per KV head g:
 * k_codes/v_codes [Hkv][L][d], s_k/s_v/lambda [Hkv][d] FP16 bits.
 * out [Hq][d] FP16 bits. */
void oracle_kv4_attention(const uint16_t *q, const int8_t *k_codes, const uint16_t *s_k,
                          const int8_t *v_codes, const uint16_t *s_v, const uint16_t *lambda,
                          int64_t Hq, int64_t Hkv, int64_t L, int64_t d, uint16_t *out)
{
    int64_t G = Hq / Hkv;
    double inv = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(static)
    for (int64_t h = 0; h < Hq; ++h) {
        int64_t g = h / G;
        const int8_t *kc = k_codes + g * L * d;
        const int8_t *vc = v_codes + g * L * d;
        double *sc = (double *)malloc(sizeof(double) * (size_t)L);
        double mx = -INFINITY;
        for (int64_t l = 0; l < L; ++l) {
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) {
                double qs = (double)oracle_half_to_float(q[h * d + c]) *
                            (double)oracle_half_to_float(lambda[g * d + c]);         /* Q' = Q lambda */
                double kh = (double)oracle_half_to_float(s_k[g * d + c]) * (double)kc[l * d + c];
                acc += qs * kh;
            }
            sc[l] = acc * inv;
            if (sc[l] > mx) mx = sc[l];
        }
        double den = 0.0;
        for (int64_t l = 0; l < L; ++l) {
            sc[l] = exp(sc[l] - mx);
            den += sc[l];
        }
        for (int64_t c = 0; c < d; ++c) {
            double num = 0.0;
            for (int64_t l = 0; l < L; ++l)
                num += sc[l] * (double)oracle_half_to_float(s_v[g * d + c]) * (double)vc[l * d + c];
            out[h * d + c] = oracle_double_to_half_rn(num / den);
        }
        free(sc);
    }
}

/* Number of OpenMP threads the parallel loops above use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets that number (n >= 1) for later calls from this thread; timing only,
 * the results do not depend on it. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
