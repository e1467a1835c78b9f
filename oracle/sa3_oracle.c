/*
 * sa3_oracle.c -- plain, slow CPU oracle for microscaled-FP4 attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, the smoke check in __graft_entry__.py and the
 * cpu_baseline / reference leg of bench.py use it.  It shares no code, header,
 * table or helper with the CUDA library; it is written from the method's
 * definition, step by step, in the order the method states them.
 *
 * Sources (pages by title, section):
 *  - "SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
 *    Acceleration" (atlas.scime.ai summary), section "Approach": K is smoothed
 *    by subtracting its mean over tokens, which leaves softmax attention
 *    unchanged.                                                   -> kmean()
 *  - "SageAttention3: Microscaling FP4 Attention for Inference and An
 *    Exploration of 8-Bit Training" (transistor.fm / mlsanity.com abstract):
 *    attention computed on Blackwell FP4 tensor cores with microscaled FP4
 *    operands.                                                    -> quantize
 *  - references listed on mlsanity.com: "FP8 Formats for Deep Learning"
 *    (E4M3 scale format) and "Microscaling Data Formats for Deep Learning"
 *    (E2M1 element format, one shared scale per small block)     -> codecs
 *  - "Online normalizer calculation for softmax" and "FlashAttention" (same
 *    reference list): blockwise softmax with a running max and a running
 *    sum.                                                         -> attn_fwd
 *
 * Fixed tiling of the method: Q blocks and KV blocks of 128 tokens; P is
 * quantized once per KV block, after the running row max has been updated
 * with that block; one E4M3 scale per 16 consecutive elements along the
 * contraction dimension (d for Q and K, tokens for V and P).
 *
 * Readings where the pages are silent (each is restated where it is used):
 *  R1 the K mean runs over the Nkv real tokens of one (batch, head); summed
 *     in fp64 in token order, divided by Nkv in fp64, rounded once to fp32;
 *  R2 K_s = fp32(K) - mean, one fp32 subtraction;
 *  R3 block scale s = E4M3_RN_satfinite(fp32(amax / 6)); r = fp32(1 / s);
 *     code = E2M1_RN_satfinite(fp32(x * r)); s == 0 gives all-zero codes;
 *  R4 E2M1 and E4M3 round to nearest, ties to even, and keep the sign of a
 *     value that rounds to zero (-0 -> code 0x8);
 *  R5 packing: element 2i in the low nibble, element 2i+1 in the high one;
 *  R6 V is quantized transposed: 16-token blocks per channel;
 *  R7 raw Q is quantized (no Q smoothing); S is scaled by
 *     c = fp32(sm_scale * log2(e)) in fp32 before the softmax, exp base 2;
 *  R8 P = exp2(t - m_new) with m_new the running max including the current
 *     block; the row sum l accumulates the unquantized P;
 *  R9 columns >= Nkv and, when causal, columns > row + Nkv - Nq are -inf
 *     before the max;
 *  R11 Q may have fewer or more tokens (Nq) than K and V (Nkv); the causal
 *     mask then aligns the last query with the last key (for Nq == Nkv this
 *     is the usual lower-triangular mask);
 *  R12 a query row that sees no key at all (causal, Nq > Nkv) outputs 0;
 *  R13 (optional) V smoothing: V_s = fp32(V) - mean of V over the keys,
 *     quantized like V; out = bf16(O / l + mean) in fp32;
 *  R14 (optional) two-level P: P' = P * 2^11 (the largest power of two with
 *     2^k / 6 <= 448, so no block scale saturates) is microscaled instead of
 *     P, and out = bf16((O / l) * 2^-11); being exact in binary, the
 *     pre-scale changes only blocks whose E4M3 scale was subnormal or 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define BLK 128   /* Q block and KV block, tokens */
#define VEC 16    /* elements per E4M3 scale */

/* ---------------------------------------------------------------- codecs */

/* E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no inf/nan. */
double oracle_e2m1_value(int code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -mag : mag;
}

/* E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits;
 * S.1111.111 is NaN, there is no infinity; largest finite value 448. */
double oracle_e4m3_value(int code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp(m / 8.0, -6);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Round to the nearest E2M1 magnitude, ties to the even code, saturating at
 * 6; the sign bit is copied from x (reading R4).  Written as a search over
 * the eight magnitudes so that it can be checked by eye. */
int oracle_e2m1_rn(float x)
{
    double a = fabs((double)x);
    /* saturation: at or above the largest magnitude the answer is 6 (for
     * huge a the two distances below would compare equal in fp64) */
    if (a >= 6.0) return (signbit(x) ? 8 : 0) | 7;
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {
        double dist = fabs(a - oracle_e2m1_value(c));
        if (dist < bestd || (dist == bestd && (c & 1) == 0)) {
            best = c;
            bestd = dist;
        }
    }
    return (signbit(x) ? 8 : 0) | best;
}

/* Round a non-negative value to the nearest finite E4M3 magnitude, ties to
 * the even code, saturating at 448 (codes 0x00..0x7E). */
int oracle_e4m3_rn_sat(float x)
{
    double a = fabs((double)x);
    if (a >= 448.0) return 0x7E; /* saturation, as for E2M1 above */
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 127; ++c) {
        double dist = fabs(a - oracle_e4m3_value(c));
        if (dist < bestd || (dist == bestd && (c & 1) == 0)) {
            best = c;
            bestd = dist;
        }
    }
    return best;
}

static float bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (on the magnitude). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lo = u & 0xFFFF0000u;
    uint32_t rem = u & 0xFFFFu;
    uint32_t hi = lo + 0x10000u;
    uint32_t r;
    if (rem > 0x8000u) r = hi;
    else if (rem < 0x8000u) r = lo;
    else r = ((lo >> 16) & 1u) ? hi : lo;
    return (uint16_t)(r >> 16);
}

/* Lookup tables filled once from the definitions above. */
static float g_e2m1[16];
static float g_e4m3[256];
static int g_tables_ready = 0;

static void tables_init(void)
{
    if (g_tables_ready) return;
    for (int c = 0; c < 16; ++c) g_e2m1[c] = (float)oracle_e2m1_value(c);
    for (int c = 0; c < 256; ++c) g_e4m3[c] = (float)oracle_e4m3_value(c);
    g_tables_ready = 1;
}

/* One 16-element block (reading R3).  x holds n <= 16 values (missing
 * tokens of a ragged last block are zeros and are passed as zeros).
 * Writes 16 codes and returns the scale byte. */
static int quant_block(const float *x, int *codes)
{
    float amax = 0.0f;
    for (int i = 0; i < VEC; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float ratio = amax / 6.0f;
    int sc = oracle_e4m3_rn_sat(ratio);
    float s = g_e4m3[sc];
    if (s == 0.0f) {
        for (int i = 0; i < VEC; ++i) codes[i] = 0;
        return sc;
    }
    float r = 1.0f / s;
    for (int i = 0; i < VEC; ++i) {
        float y = x[i] * r;
        codes[i] = oracle_e2m1_rn(y);
    }
    return sc;
}

int oracle_padded_len(int N) { return (N + BLK - 1) / BLK * BLK; }

/* ------------------------------------------------------- K smoothing (R1) */

void oracle_kmean(const uint16_t *k, int B, int H, int N, int d, float *mean)
{
    for (long bh = 0; bh < (long)B * H; ++bh) {
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int t = 0; t < N; ++t)
                acc += (double)bf16_to_f32(k[(bh * N + t) * d + c]);
            mean[bh * d + c] = (float)(acc / (double)N);
        }
    }
}

/* ----------------------------------------------------- quantization (R1-R6)
 * Q has Nq tokens, K and V have Nkv (Nq == Nkv for self-attention).
 * Canonical layouts written here (Np = a length rounded up to 128):
 *   q_codes          : [B*H][Np(Nq)][d/2]    bytes
 *   q_sf             : [B*H][Np(Nq)][d/16]   E4M3 bytes
 *   k_codes, k_sf    : the same with Np(Nkv)
 *   vt_codes         : [B*H][d][Np(Nkv)/2]   bytes (V transposed)
 *   vt_sf            : [B*H][d][Np(Nkv)/16]  E4M3 bytes
 *   k_mean           : [B*H][d] fp32, the mean over the Nkv tokens of K
 *   v_mean           : [B*H][d] fp32, the same for V (smooth_v only)
 * Padding tokens get code 0 and scale byte 0.
 * smooth_k = 0 skips the subtraction (used to measure what smoothing buys).
 * smooth_v = 1 quantizes V_s = fp32(V) - mean of V over the Nkv tokens, the
 * same recipe as K (R13); attention adds the mean back after O / l. */
static void quant_rows(const uint16_t *x_in, long bh, int N, int Np, int d, const float *sub,
                       uint8_t *codes_out, uint8_t *sf_out)
{
    float x[VEC];
    int codes[VEC];
    for (int t = 0; t < N; ++t) {
        for (int b = 0; b < d / VEC; ++b) {
            for (int i = 0; i < VEC; ++i) {
                float xv = bf16_to_f32(x_in[(bh * N + t) * d + b * VEC + i]);
                x[i] = sub ? xv - sub[b * VEC + i] : xv;  /* one fp32 subtraction (R2) */
            }
            int sc = quant_block(x, codes);
            sf_out[(bh * Np + t) * (d / VEC) + b] = (uint8_t)sc;
            for (int i = 0; i < VEC; i += 2)
                codes_out[(bh * Np + t) * (d / 2) + (b * VEC + i) / 2] = (uint8_t)(codes[i] | (codes[i + 1] << 4));
        }
    }
}

void oracle_quantize_qkv(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         int B, int H, int Nq, int Nkv, int d, int smooth_k, int smooth_v,
                         uint8_t *q_codes, uint8_t *q_sf,
                         uint8_t *k_codes, uint8_t *k_sf,
                         uint8_t *vt_codes, uint8_t *vt_sf, float *k_mean, float *v_mean)
{
    tables_init();
    const long BH = (long)B * H;
    const int Npq = oracle_padded_len(Nq);
    const int Np = oracle_padded_len(Nkv);
    oracle_kmean(k, B, H, Nkv, d, k_mean);
    if (smooth_v) oracle_kmean(v, B, H, Nkv, d, v_mean);

    memset(q_codes, 0, (size_t)BH * Npq * d / 2);
    memset(q_sf, 0, (size_t)BH * Npq * d / VEC);
    memset(k_codes, 0, (size_t)BH * Np * d / 2);
    memset(k_sf, 0, (size_t)BH * Np * d / VEC);
    memset(vt_codes, 0, (size_t)BH * d * Np / 2);
    memset(vt_sf, 0, (size_t)BH * d * Np / VEC);

#pragma omp parallel for schedule(dynamic)
    for (long bh = 0; bh < BH; ++bh) {
        float x[VEC];
        int codes[VEC];
        /* Q and K: blocks of 16 along d, per token; K smoothed (R2). */
        quant_rows(q, bh, Nq, Npq, d, NULL, q_codes, q_sf);
        quant_rows(k, bh, Nkv, Np, d, smooth_k ? k_mean + bh * d : NULL, k_codes, k_sf);
        /* V: blocks of 16 tokens, per channel (R6). */
        for (int c = 0; c < d; ++c) {
            for (int tb = 0; tb < Np / VEC; ++tb) {
                for (int i = 0; i < VEC; ++i) {
                    int t = tb * VEC + i;
                    float vv = (t < Nkv) ? bf16_to_f32(v[(bh * Nkv + t) * d + c]) : 0.0f;
                    x[i] = (t < Nkv && smooth_v) ? vv - v_mean[bh * d + c] : vv;
                }
                int sc = quant_block(x, codes);
                vt_sf[(bh * d + c) * (Np / VEC) + tb] = (uint8_t)sc;
                for (int i = 0; i < VEC; i += 2)
                    vt_codes[(bh * d + c) * (Np / 2) + (tb * VEC + i) / 2] =
                        (uint8_t)(codes[i] | (codes[i + 1] << 4));
            }
        }
    }
}

/* Dequantize one packed element. */
static double deq(const uint8_t *codes, const uint8_t *sf, long elem, long sf_idx)
{
    uint8_t byte = codes[elem >> 1];
    int code = (elem & 1) ? (byte >> 4) : (byte & 15);
    return (double)g_e2m1[code] * (double)g_e4m3[sf[sf_idx]];
}

/* ------------------------------------------------- tiled attention (R7-R9)
 * Nq query rows, Nkv key/value columns.  causal masks col > row + Nkv - Nq
 * (the last query row aligned with the last key, R11); a row that sees no
 * column at all gets output 0 (R12).
 * p_two_level: P is scaled by 2^11 before it is microscaled and the output
 * by 2^-11 after O / l (R14); v_mean (NULL: none) is added after O / l (R13).
 * units: n_units pairs (bh, q_block); NULL means every (bh, q_block).
 * out: bf16 [B*H][Nq][d]; only rows of the listed units are written.
 * out32 (NULL: not wanted): the same outputs in fp32 just before the final
 * bf16 rounding, so that a test can tell a value sitting on a bf16
 * rounding tie from a wrong one. */
void oracle_attn_fwd(const uint8_t *q_codes, const uint8_t *q_sf,
                     const uint8_t *k_codes, const uint8_t *k_sf,
                     const uint8_t *vt_codes, const uint8_t *vt_sf,
                     int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                     int p_two_level, const float *v_mean,
                     const int32_t *units, int n_units, uint16_t *out, float *out32)
{
    tables_init();
    const float p_pre = p_two_level ? 2048.0f : 1.0f;   /* 2^11, exact (R14) */
    const long BH = (long)B * H;
    const int Npq = oracle_padded_len(Nq);
    const int Np = oracle_padded_len(Nkv);
    const int nqb = Npq / BLK;
    const int off = Nkv - Nq;
    const float c_log2 = (float)((double)sm_scale * 1.4426950408889634);
    const long total = units ? n_units : BH * nqb;

#pragma omp parallel for schedule(dynamic)
    for (long u = 0; u < total; ++u) {
        long bh = units ? units[2 * u] : u / nqb;
        int qb = units ? units[2 * u + 1] : (int)(u % nqb);
        /* KV blocks up to the last column any row of this Q block sees */
        int nkv = Np / BLK;
        if (causal) {
            int last = qb * BLK + BLK - 1 + off;
            int nb = last < 0 ? 0 : last / BLK + 1;
            if (nb < nkv) nkv = nb;
        }
        int ncol = nkv * BLK;
        /* Dequantized operands of this (batch, head), cached so that each
         * value is decoded once; the sums below are unchanged by this. */
        double *qrow = (double *)malloc(sizeof(double) * d);
        double *khat = (double *)malloc(sizeof(double) * ((size_t)ncol * d + 1));
        double *vhat = (double *)malloc(sizeof(double) * ((size_t)ncol * d + 1));
        float *O = (float *)malloc(sizeof(float) * d);
        float t[BLK], p[BLK], phat[BLK];
        int codes[VEC];
        for (int col = 0; col < ncol; ++col)
            for (int c = 0; c < d; ++c)
                khat[(size_t)col * d + c] = deq(k_codes, k_sf, (bh * Np + col) * d + c,
                                                (bh * Np + col) * (d / VEC) + c / VEC);
        for (int c = 0; c < d; ++c)
            for (int col = 0; col < ncol; ++col)
                vhat[(size_t)c * ncol + col] = deq(vt_codes, vt_sf, (bh * d + c) * Np + col,
                                                   (bh * d + c) * (Np / VEC) + col / VEC);

        for (int row = qb * BLK; row < qb * BLK + BLK && row < Nq; ++row) {
            for (int c = 0; c < d; ++c)
                qrow[c] = deq(q_codes, q_sf, (bh * Npq + row) * d + c,
                              (bh * Npq + row) * (d / VEC) + c / VEC);
            float m = -INFINITY, l = 0.0f;
            for (int c = 0; c < d; ++c) O[c] = 0.0f;

            for (int j = 0; j < nkv; ++j) {
                /* S row for this KV block: exact fp64 dot, rounded once. */
                float bmax = -INFINITY;
                for (int i = 0; i < BLK; ++i) {
                    int col = j * BLK + i;
                    if (col >= Nkv || (causal && col > row + off)) { t[i] = -INFINITY; continue; }
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c)
                        acc += qrow[c] * khat[(size_t)col * d + c];
                    float s = (float)acc;
                    t[i] = s * c_log2;
                    if (t[i] > bmax) bmax = t[i];
                }
                /* Online softmax update. */
                float m_new = m > bmax ? m : bmax;
                float alpha, rowsum;
                if (m_new == -INFINITY) { /* fully masked so far (R9 guard) */
                    alpha = 1.0f;
                    for (int i = 0; i < BLK; ++i) p[i] = 0.0f;
                } else {
                    alpha = exp2f(m - m_new);
                    for (int i = 0; i < BLK; ++i) p[i] = exp2f(t[i] - m_new);
                }
                double psum = 0.0;
                for (int i = 0; i < BLK; ++i) psum += p[i];
                rowsum = (float)psum;
                l = alpha * l + rowsum;
                /* Quantize P per 16-column block (R3, R8), after the exact
                 * two-level pre-scale when asked for (R14). */
                float pp[BLK];
                for (int i = 0; i < BLK; ++i) pp[i] = p[i] * p_pre;
                for (int b = 0; b < BLK / VEC; ++b) {
                    int sc = quant_block(pp + b * VEC, codes);
                    for (int i = 0; i < VEC; ++i)
                        phat[b * VEC + i] = g_e2m1[codes[i]] * g_e4m3[sc];
                }
                /* O = alpha * O + P^ V^ (exact fp64 sum, rounded once). */
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int i = 0; i < BLK; ++i)
                        acc += (double)phat[i] * vhat[(size_t)c * ncol + j * BLK + i];
                    O[c] = alpha * O[c] + (float)acc;
                }
                m = m_new;
            }
            for (int c = 0; c < d; ++c) {
                if (!(l > 0.0f)) {
                    out[(bh * Nq + row) * d + c] = 0;
                    if (out32) out32[(bh * Nq + row) * d + c] = 0.0f;
                    continue;
                }
                float o = O[c] / l;
                if (p_two_level) o = o * (1.0f / 2048.0f);  /* exact */
                if (v_mean) o = o + v_mean[bh * d + c];
                out[(bh * Nq + row) * d + c] = oracle_f32_to_bf16(o);
                if (out32) out32[(bh * Nq + row) * d + c] = o;
            }
        }
        free(qrow);
        free(khat);
        free(vhat);
        free(O);
    }
}

/* --------------------------------------------- exact attention (fp64)
 * softmax(Q K^T * sm_scale) V on the bf16 inputs, no quantization, with the
 * masks of oracle_attn_fwd.  k_sub, if not NULL, is subtracted from K first
 * (fp32 [B*H][d]); this is how the smoothing invariance is checked.  Rows
 * of the listed units only; a row that sees no column gets 0. */
void oracle_attn_exact(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                       const float *k_sub, const int32_t *units, int n_units,
                       double *out)
{
    const long BH = (long)B * H;
    const int nqb = oracle_padded_len(Nq) / BLK;
    const int off = Nkv - Nq;
    const long total = units ? n_units : BH * nqb;

#pragma omp parallel for schedule(dynamic)
    for (long u = 0; u < total; ++u) {
        long bh = units ? units[2 * u] : u / nqb;
        int qb = units ? units[2 * u + 1] : (int)(u % nqb);
        double *logit = (double *)malloc(sizeof(double) * (Nkv + 1));
        for (int row = qb * BLK; row < qb * BLK + BLK && row < Nq; ++row) {
            int ncol = causal ? row + off + 1 : Nkv;
            if (ncol > Nkv) ncol = Nkv;
            if (ncol <= 0) {
                for (int c = 0; c < d; ++c) out[(bh * Nq + row) * d + c] = 0.0;
                continue;
            }
            double mx = -INFINITY;
            for (int col = 0; col < ncol; ++col) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) {
                    double kk = bf16_to_f32(k[(bh * Nkv + col) * d + c]);
                    if (k_sub) kk -= (double)k_sub[bh * d + c];
                    acc += (double)bf16_to_f32(q[(bh * Nq + row) * d + c]) * kk;
                }
                logit[col] = acc * (double)sm_scale;
                if (logit[col] > mx) mx = logit[col];
            }
            double den = 0.0;
            for (int col = 0; col < ncol; ++col) {
                logit[col] = exp(logit[col] - mx);
                den += logit[col];
            }
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int col = 0; col < ncol; ++col)
                    acc += logit[col] * (double)bf16_to_f32(v[(bh * Nkv + col) * d + c]);
                out[(bh * Nq + row) * d + c] = acc / den;
            }
        }
        free(logit);
    }
}

/* ===================================================== 8-bit variant
 * "SageAttention: Accurate 8-Bit Attention for Plug-and-play Inference
 * Acceleration" (summary, "Approach"): Q and K quantized to INT8 with
 * per-block scales after K is smoothed; P and V kept in FP16.  Readings
 * (I1-I5, where the summary is silent):
 *  I1 a block is one 128-token tile of Q or of K (the tiling above) over all
 *     d channels: s = fp32(amax / 127), r = fp32(1 / s), code =
 *     clamp(round_half_even(fp32(x * r)), -127, 127); s == 0 gives codes 0;
 *  I2 V is converted to FP16 (round to nearest even), stored transposed;
 *  I3 t = fp32(fp32(S) * f) with S the exact integer dot product and
 *     f = fp32(fp32(s_q * s_k) * c), c = fp32(sm_scale * log2 e);
 *  I4 P = exp2(t - m') as in R8, converted to FP16 (nearest even) before
 *     P V; the row sum l accumulates the fp32 P;
 *  I5 O accumulates in fp32 (the summary's ablation finds an FP16
 *     accumulator changes nothing; fp32 is the tensor core's native one).
 *  I6 the forward used for training ("SageAttention3: Microscaling FP4
 *     Attention for Inference and An Exploration of 8-Bit Training",
 *     abstract: 8-bit attention in the forward and backward passes) also
 *     returns, per query row, the natural-log log-sum-exp of the row's
 *     scaled logits, which a backward pass needs to rebuild P:
 *     lse = ln 2 * (m + log2 l), evaluated in fp64 from the final fp32
 *     running max m (base-2 units) and row sum l; +inf for a row that sees
 *     no key, so that exp(s - lse) is 0 there.
 * Masks, lengths and the empty-row rule are those of R9, R11, R12. */

/* fp32 -> fp16 bits, round to nearest even, overflow to inf. */
uint16_t oracle_f32_to_f16(float x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs((double)x);
    if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                          /* a = m * 2^e, m in [0.5, 1) */
    int qexp = (e - 1 >= -14) ? e - 11 : -24;  /* ulp: 10 fraction bits, or the subnormal step */
    double v = nearbyint(ldexp(a, -qexp));  /* ties to even (default rounding mode) */
    v = ldexp(v, qexp);
    if (v > 65504.0) return (uint16_t)(sign | 0x7C00u);
    if (v < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)ldexp(v, 24));  /* subnormal */
    frexp(v, &e);
    int ex = e - 1;                        /* v = 1.f * 2^ex */
    uint16_t frac = (uint16_t)(ldexp(v, -ex) * 1024.0 - 1024.0);
    return (uint16_t)(sign | ((uint16_t)(ex + 15) << 10) | frac);
}

static float f16_to_f32(uint16_t h)
{
    int ex = (h >> 10) & 31, fr = h & 1023;
    double v = ex == 0 ? ldexp((double)fr, -24) : ldexp(1024.0 + fr, ex - 25);
    if (ex == 31) v = fr ? NAN : INFINITY;
    return (float)((h & 0x8000u) ? -v : v);
}

/* INT8 codes of n values with one scale (I1); returns the scale. */
static float quant_block_i8(const float *x, int n, int8_t *codes)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float s = amax / 127.0f;
    if (s == 0.0f) {
        for (int i = 0; i < n; ++i) codes[i] = 0;
        return 0.0f;
    }
    float r = 1.0f / s;
    for (int i = 0; i < n; ++i) {
        float y = x[i] * r;
        float c = nearbyintf(y);
        if (c > 127.0f) c = 127.0f;
        if (c < -127.0f) c = -127.0f;
        codes[i] = (int8_t)c;
    }
    return s;
}

/* Layouts: q_i8 [B*H][Np(Nq)][d], q_scale [B*H][Np(Nq)/128] fp32; k_i8,
 * k_scale the same over Np(Nkv); vt_f16 [B*H][d][Np(Nkv)] fp16 bits;
 * k_mean [B*H][d].  Padding tokens: code 0, fp16 0. */
void oracle_quantize_qkv_i8(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            int B, int H, int Nq, int Nkv, int d,
                            int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale,
                            uint16_t *vt_f16, float *k_mean)
{
    const long BH = (long)B * H;
    const int Npq = oracle_padded_len(Nq), Np = oracle_padded_len(Nkv);
    oracle_kmean(k, B, H, Nkv, d, k_mean);
    memset(q_i8, 0, (size_t)BH * Npq * d);
    memset(k_i8, 0, (size_t)BH * Np * d);
    memset(vt_f16, 0, (size_t)BH * d * Np * 2);
#pragma omp parallel for schedule(dynamic)
    for (long bh = 0; bh < BH; ++bh) {
        float *x = (float *)malloc(sizeof(float) * BLK * d);
        for (int which = 0; which < 2; ++which) {
            const uint16_t *src = which ? k : q;
            const int N = which ? Nkv : Nq, Npx = which ? Np : Npq;
            int8_t *codes = which ? k_i8 : q_i8;
            float *scale = which ? k_scale : q_scale;
            for (int tb = 0; tb < Npx / BLK; ++tb) {
                int n = 0;
                for (int t = tb * BLK; t < tb * BLK + BLK && t < N; ++t)
                    for (int c = 0; c < d; ++c) {
                        float xv = bf16_to_f32(src[(bh * N + t) * d + c]);
                        x[n++] = which ? xv - k_mean[bh * d + c] : xv;  /* K smoothed (R2) */
                    }
                scale[bh * (Npx / BLK) + tb] = quant_block_i8(x, n, codes + (bh * Npx + (long)tb * BLK) * d);
            }
        }
        for (int c = 0; c < d; ++c)
            for (int t = 0; t < Nkv; ++t)
                vt_f16[(bh * d + c) * Np + t] = oracle_f32_to_f16(bf16_to_f32(v[(bh * Nkv + t) * d + c]));
        free(x);
    }
}

void oracle_attn_fwd_i8(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8, const float *k_scale,
                        const uint16_t *vt_f16, int B, int H, int Nq, int Nkv, int d, int causal,
                        float sm_scale, const int32_t *units, int n_units, uint16_t *out, float *lse)
{
    const long BH = (long)B * H;
    const int Npq = oracle_padded_len(Nq), Np = oracle_padded_len(Nkv);
    const int nqb = Npq / BLK, off = Nkv - Nq;
    const float c_log2 = (float)((double)sm_scale * 1.4426950408889634);
    const long total = units ? n_units : BH * nqb;

#pragma omp parallel for schedule(dynamic)
    for (long u = 0; u < total; ++u) {
        long bh = units ? units[2 * u] : u / nqb;
        int qb = units ? units[2 * u + 1] : (int)(u % nqb);
        int nkv = Np / BLK;
        if (causal) {
            int last = qb * BLK + BLK - 1 + off;
            int nb = last < 0 ? 0 : last / BLK + 1;
            if (nb < nkv) nkv = nb;
        }
        float *O = (float *)malloc(sizeof(float) * d);
        /* FP16 V of this (batch, head), decoded once */
        float *vhat = (float *)malloc(sizeof(float) * ((size_t)d * nkv * BLK + 1));
        for (int c = 0; c < d; ++c)
            for (int col = 0; col < nkv * BLK; ++col)
                vhat[(size_t)c * nkv * BLK + col] = f16_to_f32(vt_f16[(bh * d + c) * Np + col]);
        float t[BLK], p[BLK], p16[BLK];
        for (int row = qb * BLK; row < qb * BLK + BLK && row < Nq; ++row) {
            const int8_t *qr = q_i8 + (bh * Npq + row) * d;
            float m = -INFINITY, l = 0.0f;
            for (int c = 0; c < d; ++c) O[c] = 0.0f;
            for (int j = 0; j < nkv; ++j) {
                const float f = (q_scale[bh * nqb + qb] * k_scale[bh * (Np / BLK) + j]) * c_log2;  /* I3 */
                float bmax = -INFINITY;
                for (int i = 0; i < BLK; ++i) {
                    int col = j * BLK + i;
                    if (col >= Nkv || (causal && col > row + off)) { t[i] = -INFINITY; continue; }
                    const int8_t *kr = k_i8 + (bh * Np + col) * d;
                    long acc = 0;
                    for (int c = 0; c < d; ++c) acc += (long)qr[c] * kr[c];
                    t[i] = (float)acc * f;
                    if (t[i] > bmax) bmax = t[i];
                }
                float m_new = m > bmax ? m : bmax;
                float alpha;
                if (m_new == -INFINITY) {
                    alpha = 1.0f;
                    for (int i = 0; i < BLK; ++i) p[i] = 0.0f;
                } else {
                    alpha = exp2f(m - m_new);
                    for (int i = 0; i < BLK; ++i) p[i] = exp2f(t[i] - m_new);
                }
                double psum = 0.0;
                for (int i = 0; i < BLK; ++i) psum += p[i];
                l = alpha * l + (float)psum;
                for (int i = 0; i < BLK; ++i) p16[i] = f16_to_f32(oracle_f32_to_f16(p[i]));  /* I4 */
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int i = 0; i < BLK; ++i)
                        acc += (double)p16[i] * (double)vhat[(size_t)c * nkv * BLK + j * BLK + i];
                    O[c] = alpha * O[c] + (float)acc;
                }
                m = m_new;
            }
            for (int c = 0; c < d; ++c)
                out[(bh * Nq + row) * d + c] = l > 0.0f ? oracle_f32_to_bf16(O[c] / l) : 0;
            if (lse)  /* I6 */
                lse[bh * Nq + row] = l > 0.0f ? (float)(0.69314718055994531 * ((double)m + log2((double)l)))
                                              : INFINITY;
        }
        free(O);
        free(vhat);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
