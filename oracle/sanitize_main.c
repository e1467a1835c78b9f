/*
 * sanitize_main.c -- TEST INFRASTRUCTURE ONLY: a driver that runs every entry
 * point of sa3_oracle.c on small seeded inputs, so that the oracle can be
 * built with the host's address and undefined-behaviour sanitizers
 * (tests/test_oracle_sanitizers.py).  Shapes cover ragged tails, one-token
 * and decode-sized queries, more queries than keys, both masks, d = 64 and
 * 128, the optional terms (two-level P, V smoothing, log-sum-exp) and
 * sampled work units.  Every output buffer is allocated to its exact size,
 * so any out-of-range write or read is reported.  Exit status 0 when every
 * call returns and every output is finite.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int oracle_padded_len(int N);
double oracle_e2m1_value(int code);
double oracle_e4m3_value(int code);
int oracle_e2m1_rn(float x);
int oracle_e4m3_rn_sat(float x);
uint16_t oracle_f32_to_bf16(float f);
uint16_t oracle_f32_to_f16(float x);
void oracle_kmean(const uint16_t *k, int B, int H, int N, int d, float *mean);
void oracle_quantize_qkv(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int H, int Nq, int Nkv,
                         int d, int smooth_k, int smooth_v, uint8_t *q_codes, uint8_t *q_sf, uint8_t *k_codes,
                         uint8_t *k_sf, uint8_t *vt_codes, uint8_t *vt_sf, float *k_mean, float *v_mean);
void oracle_attn_fwd(const uint8_t *q_codes, const uint8_t *q_sf, const uint8_t *k_codes, const uint8_t *k_sf,
                     const uint8_t *vt_codes, const uint8_t *vt_sf, int B, int H, int Nq, int Nkv, int d, int causal,
                     float sm_scale, int p_two_level, const float *v_mean, const int32_t *units, int n_units,
                     uint16_t *out, float *out32);
void oracle_attn_exact(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int H, int Nq, int Nkv, int d,
                       int causal, float sm_scale, const float *k_sub, const int32_t *units, int n_units,
                       double *out);
void oracle_quantize_qkv_i8(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int H, int Nq, int Nkv,
                            int d, int8_t *q_i8, float *q_scale, int8_t *k_i8, float *k_scale, uint16_t *vt_f16,
                            float *k_mean);
void oracle_attn_fwd_i8(const int8_t *q_i8, const float *q_scale, const int8_t *k_i8, const float *k_scale,
                        const uint16_t *vt_f16, int B, int H, int Nq, int Nkv, int d, int causal, float sm_scale,
                        const int32_t *units, int n_units, uint16_t *out, float *lse);

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;

/* xorshift64*: a uniform float in [-2, 2), rounded to bf16 */
static uint16_t rand_bf16(void)
{
    rng_state ^= rng_state >> 12;
    rng_state ^= rng_state << 25;
    rng_state ^= rng_state >> 27;
    const uint64_t r = rng_state * 0x2545F4914F6CDD1Dull;
    const float x = (float)((double)(r >> 11) * 0x1.0p-53 * 4.0 - 2.0);
    return oracle_f32_to_bf16(x);
}

static void *alloc(size_t n)
{
    void *p = malloc(n ? n : 1);
    if (!p) {
        fprintf(stderr, "out of memory\n");
        exit(2);
    }
    return p;
}

static int finite_bf16(const uint16_t *x, size_t n)
{
    for (size_t i = 0; i < n; ++i)
        if ((x[i] & 0x7F80u) == 0x7F80u) return 0;
    return 1;
}

static int run_case(int B, int H, int Nq, int Nkv, int d)
{
    const long BH = (long)B * H;
    const int Npq = oracle_padded_len(Nq), Np = oracle_padded_len(Nkv);
    const size_t nq = (size_t)BH * Nq * d, nkv = (size_t)BH * Nkv * d;
    uint16_t *q = alloc(nq * 2), *k = alloc(nkv * 2), *v = alloc(nkv * 2);
    for (size_t i = 0; i < nq; ++i) q[i] = rand_bf16();
    for (size_t i = 0; i < nkv; ++i) k[i] = rand_bf16();
    for (size_t i = 0; i < nkv; ++i) v[i] = rand_bf16();
    const float sm = (float)(1.0 / sqrt((double)d));
    int ok = 1;

    /* FP4 path: quantizer with and without V smoothing, attention with every option */
    uint8_t *qc = alloc((size_t)BH * Npq * d / 2), *qs = alloc((size_t)BH * Npq * d / 16);
    uint8_t *kc = alloc((size_t)BH * Np * d / 2), *ks = alloc((size_t)BH * Np * d / 16);
    uint8_t *vc = alloc((size_t)BH * d * Np / 2), *vs = alloc((size_t)BH * d * Np / 16);
    float *km = alloc((size_t)BH * d * 4), *vm = alloc((size_t)BH * d * 4);
    uint16_t *out = alloc(nq * 2);
    float *out32 = alloc(nq * 4);
    for (int smooth_v = 0; smooth_v < 2; ++smooth_v) {
        oracle_quantize_qkv(q, k, v, B, H, Nq, Nkv, d, 1, smooth_v, qc, qs, kc, ks, vc, vs, km, smooth_v ? vm : NULL);
        for (int causal = 0; causal < 2; ++causal)
            for (int two = 0; two < 2; ++two) {
                memset(out, 0, nq * 2);
                oracle_attn_fwd(qc, qs, kc, ks, vc, vs, B, H, Nq, Nkv, d, causal, sm, two, smooth_v ? vm : NULL,
                                NULL, 0, out, out32);
                ok &= finite_bf16(out, nq);
            }
    }
    /* sampled units: the last Q block of the last head, then the first */
    const int32_t units[4] = {(int32_t)(BH - 1), Npq / 128 - 1, 0, 0};
    oracle_attn_fwd(qc, qs, kc, ks, vc, vs, B, H, Nq, Nkv, d, 1, sm, 0, NULL, units, 2, out, NULL);
    ok &= finite_bf16(out, nq);

    /* exact attention, with and without the K mean subtracted */
    double *ex = alloc(nq * 8);
    oracle_attn_exact(q, k, v, B, H, Nq, Nkv, d, 1, sm, km, NULL, 0, ex);
    oracle_attn_exact(q, k, v, B, H, Nq, Nkv, d, 0, sm, NULL, units, 2, ex);
    for (size_t i = 0; i < nq; ++i) ok &= isfinite(ex[i]) != 0;

    /* 8-bit variant, with and without the log-sum-exp */
    int8_t *q8 = alloc((size_t)BH * Npq * d), *k8 = alloc((size_t)BH * Np * d);
    float *qsc = alloc((size_t)BH * (Npq / 128) * 4), *ksc = alloc((size_t)BH * (Np / 128) * 4);
    uint16_t *vt16 = alloc((size_t)BH * d * Np * 2);
    float *lse = alloc((size_t)BH * Nq * 4);
    oracle_quantize_qkv_i8(q, k, v, B, H, Nq, Nkv, d, q8, qsc, k8, ksc, vt16, km);
    for (int causal = 0; causal < 2; ++causal) {
        oracle_attn_fwd_i8(q8, qsc, k8, ksc, vt16, B, H, Nq, Nkv, d, causal, sm, NULL, 0, out, lse);
        ok &= finite_bf16(out, nq);
        for (size_t i = 0; i < (size_t)BH * Nq; ++i) ok &= !isnan(lse[i]);
        oracle_attn_fwd_i8(q8, qsc, k8, ksc, vt16, B, H, Nq, Nkv, d, causal, sm, units, 2, out, NULL);
    }

    free(q), free(k), free(v), free(qc), free(qs), free(kc), free(ks), free(vc), free(vs), free(km), free(vm);
    free(out), free(out32), free(ex), free(q8), free(k8), free(qsc), free(ksc), free(vt16), free(lse);
    if (!ok) fprintf(stderr, "non-finite output: B=%d H=%d Nq=%d Nkv=%d d=%d\n", B, H, Nq, Nkv, d);
    return ok;
}

int main(void)
{
    static const int shapes[][5] = {
        {1, 2, 1, 1, 64},    {1, 2, 15, 15, 64},  {1, 2, 129, 129, 64}, {1, 1, 77, 300, 64},
        {1, 2, 300, 130, 64}, {2, 1, 1, 257, 128}, {1, 2, 200, 200, 128}, {1, 1, 260, 17, 128},
    };
    int ok = 1;
    for (size_t i = 0; i < sizeof shapes / sizeof shapes[0]; ++i)
        ok &= run_case(shapes[i][0], shapes[i][1], shapes[i][2], shapes[i][3], shapes[i][4]);
    /* scalar codecs over their whole input ranges */
    double acc = 0.0;
    for (int c = 0; c < 16; ++c) acc += oracle_e2m1_value(c);
    for (int c = 0; c < 256; ++c) acc += fabs(oracle_e4m3_value(c)) < 1e9 ? 0.0 : 1.0;
    for (int i = -4000; i <= 4000; ++i) {
        const float x = (float)i / 256.0f;
        acc += oracle_e2m1_rn(x) + oracle_e4m3_rn_sat(x * 64.0f) + oracle_f32_to_f16(x * 1e3f);
    }
    if (!isfinite(acc)) ok = 0;
    printf(ok ? "ok\n" : "failed\n");
    return ok ? 0 : 1;
}
