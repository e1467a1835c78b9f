// probe.cuh -- throughput probe of the block-scaled FP4 tensor-core MMA.
//
// Not a step of the method: it measures the rate that the attention
// kernel's two products (S = Q^ K^T and O += P^ V^, both
// tcgen05.mma.kind::mxf4nvf4.block_scale.scale_vec::4X with M = 128) can
// reach on this part, as the denominator of the attention roofline.  One
// CTA per SM issues `iters` MMAs of M = 128, N = kN, K = 64 from shared
// memory into one TMEM accumulator.  Every code is E2M1 1.0 and every scale
// E4M3 1.0, so each MMA adds exactly 64 to every accumulator element: after
// the loop each element must read 64 * iters (exact in fp32 for iters <=
// 2^18), which the caller checks.
#pragma once

#include "sa3_internal.h"
#include "sm100.cuh"

namespace sa3 {
namespace probe {

constexpr int kThreads = 128;
constexpr int kSmemBytes = 120 * 1024;  // forces one CTA per SM (two would not fit)

template <int kN>
__global__ void __launch_bounds__(kThreads, 1) fp4_mma_rate_kernel(int iters, float *out) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_s - raw_s);
    // A: 128 rows x 32 bytes; B: kN rows x 32 bytes (K = 64 E2M1 codes per
    // row, 32-byte swizzle: every byte is the same, so the swizzle does not
    // matter); scale atoms: 512 bytes per 128 rows.
    constexpr int oA = 0, oB = 4096, oSfa = oB + kN * 32, oSfb = oSfa + 512, oBar = oSfb + 1024;
    uint64_t *bar = reinterpret_cast<uint64_t *>(base + oBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    for (int i = threadIdx.x; i < oSfa / 4; i += kThreads) reinterpret_cast<uint32_t *>(base)[i] = 0x22222222u;
    for (int i = threadIdx.x; i < 1536 / 4; i += kThreads)
        reinterpret_cast<uint32_t *>(base + oSfa)[i] = 0x38383838u;  // E4M3 1.0
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_d = tmem, t_sfa = tmem + 256, t_sfb = tmem + 260;
    if (threadIdx.x == 0) {
        tc_cp_32x128b_warpx4(t_sfa, sdesc_sf_atom(base_s + oSfa));
        for (int a = 0; a < 3; ++a) tc_cp_32x128b_warpx4(t_sfb + 4 * a, sdesc_sf_atom(base_s + oSfb + 512 * (a & 1)));
        constexpr uint32_t idesc = idesc_mxf4nvf4(128, kN);
        const uint64_t adesc = sdesc_kmajor_sw(base_s + oA, 256, 6);
        const uint64_t bdesc = sdesc_kmajor_sw(base_s + oB, 256, 6);
        for (int it = 0; it < iters; ++it) tc_mma_mxf4nvf4(t_d, adesc, bdesc, idesc, t_sfa, t_sfb, it > 0);
        tc_commit(bar);
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, abort_flag));
    tc_fence_after();
    if (ok) {
        // lane = row 32*warp + lane; read column 0 and column kN-1
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16), v);
        tmem_ld_wait();
        reg_fence32(v);
        uint32_t w[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + kN - 32, w);
        tmem_ld_wait();
        reg_fence32(w);
        // out[2*cta]: the smallest of D[:, 0]; out[2*cta+1]: the largest of D[:, kN-1]
        float lo = __uint_as_float(v[0]), hi = __uint_as_float(w[31]);
        for (int off = 16; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        float *red = reinterpret_cast<float *>(base + oBar + 64);
        if ((threadIdx.x & 31) == 0) {
            red[warp] = lo;
            red[4 + warp] = hi;
        }
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            out[2 * blockIdx.x] = fminf(fminf(red[0], red[1]), fminf(red[2], red[3]));
            out[2 * blockIdx.x + 1] = fmaxf(fmaxf(red[4], red[5]), fmaxf(red[6], red[7]));
        }
    } else {
        tc_fence_before();
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

template <int kN>
cudaError_t launch(int ctas, int iters, float *out, cudaStream_t stream) {
    cudaError_t e = smem_attr_once<fp4_mma_rate_kernel<kN>>(kSmemBytes);
    if (e != cudaSuccess) return e;
    fp4_mma_rate_kernel<kN><<<ctas, kThreads, kSmemBytes, stream>>>(iters, out);
    return cudaGetLastError();
}

}  // namespace probe
}  // namespace sa3
