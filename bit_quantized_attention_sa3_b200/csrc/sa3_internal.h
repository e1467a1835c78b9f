// sa3_internal.h -- launch parameters shared by the host API and kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sa3 {


// Q, K and V themselves reach the quantizer as TMA tensor maps.
struct QuantParams {
    uint8_t *q_fp4;
    uint8_t *q_sf;
    uint8_t *k_fp4;
    uint8_t *k_sf;
    uint8_t *vt_fp4;
    uint8_t *vt_sf;
    float *k_mean;
    float *q_scale;  // 8-bit variant: one fp32 scale per 128-token tile of Q
    float *k_scale;  // ... and of K (codes then go to q_fp4 / k_fp4 as int8, V to vt_fp4 as fp16)
    double *part;    // [BH][nchunk][d] scratch: fp64 column sums of K per chunk
    int BH;
    int N;       // K and V tokens
    int Np;      // N rounded up to 128
    int Nq;      // Q tokens (== N for self-attention)
    int Npq;     // Nq rounded up to 128
    int nchunk;  // fp64 partial sums of K per (b, h)
    int chunk;   // tokens per partial sum
    int st32;    // 1: the code outputs are 32-byte aligned, so tiles store 32-byte pieces in one instruction
};

struct AttnParams {
    const uint8_t *q_sf;
    const uint8_t *k_sf;
    const uint8_t *vt_sf;
    const float *q_scale;  // 8-bit variant: fp32 scale per 128-token tile of Q
    const float *k_scale;  // ... and of K
    __nv_bfloat16 *out;
    float *lse;        // 8-bit variant: per-row log-sum-exp (natural log), or null
    int BH;
    int N;             // key / value tokens
    int Np;            // N rounded up to 128
    int Nq;            // query tokens (== N for self-attention)
    int Npq;           // Nq rounded up to 128
    int causal;        // mask col > row + N - Nq
    float scale_log2;  // fp32(sm_scale * log2 e)
    float p_pre_log2;  // 0, or 11 for two-level P (P scaled by 2^11 before microscaling;
                       // selects the kernel instance, whose exponent is fixed)
    int npairs;        // Q-tile pairs per head (set by the launcher)
    int pair_units;    // work units that are pairs; the rest are single tiles
};

}  // namespace sa3
