// sa3_internal.h -- launch parameters shared by the host API and kernels.
#pragma once

#include <atomic>
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
    double *vpart;   // ... and of V (V smoothing only)
    float *v_mean;   // V smoothing: fp32 [BH][d] mean of V (else unused)
    int vsmooth;     // 1: V is smoothed like K (its tiles move to the second launch)
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
    const float *v_mean;  // FP4, V smoothing: fp32 [BH][d] mean of V added to every output row, or null
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
    int q_load;        // FP4: 1 = Q arrives as bf16 (3-D tensor map) and is quantized in the kernel
    int npairs;        // Q-tile pairs per head (set by the launcher)
    int pair_units;    // work units that are pairs; the rest are single tiles
};

// The two host helpers below keep per-process caches in function-local
// statics.  They have internal linkage: as inline functions of namespace
// scope the compiler would export those statics as process-wide unique
// symbols, and two builds of this library loaded into one process would then
// share them (the second build would skip raising its own kernels' limit).
namespace {

// Host: raise Kernel's dynamic shared memory limit once per device (the
// attribute persists in the device's module), so that later calls -- those
// recorded into a CUDA graph included -- make no attribute call.  Devices
// 64 and up are set on every call.
template <auto Kernel>
inline cudaError_t smem_attr_once(int bytes) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t{1} << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Host: SM count of the current device (queried once per device; 148 if the
// query fails).
inline int sm_count() {
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace

}  // namespace sa3
