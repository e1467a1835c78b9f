// quant.cu -- K smoothing and FP4 microscaling of Q, K and V.
//
// Method: "SageAttention: Accurate 8-Bit Attention for Plug-and-play
// Inference Acceleration" (summary, section "Approach") smooths K by
// subtracting its mean over tokens; "SageAttention3: Microscaling FP4
// Attention ..." (abstract) runs attention on microscaled FP4 operands:
// E2M1 codes with one E4M3 scale per 16 elements.  The exact recipe of one
// block (x_0..x_15):  s = E4M3_RN_sat(amax/6), r = 1/s, code_i =
// E2M1_RN_sat(x_i * r), all zero if s == 0 -- see include/sa3.h.
//
// HBM-bound streaming work, three launches on the caller's stream:
//   A  Q tiles, V tiles (transposed through shared memory), and fp64
//      partial sums of K over at most 16 token chunks per (b, h), ordered so
//      that K is read last;
//   B  K tiles: each CTA first adds its (b, h)'s partial sums in chunk order
//      (fp64) into the mean, then smooths and quantizes its tile (K re-read,
//      from L2 when it fits).
// Q/K tiles: two threads per 16-element block, one 128-bit load each,
// block amax combined with one warp shuffle.  V tiles: a 128-token tile
// is staged in shared memory with a 16-byte XOR swizzle so that the
// column reads of the transpose are conflict-free.
#pragma once

#include "sa3_internal.h"
#include "sm100.cuh"

namespace sa3 {

namespace {

constexpr int kTile = 128;    // tokens per Q/K/V tile
constexpr int kThreads = 256;  // threads per quantizer CTA

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void bf16x8(const uint4 &v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Byte offset of scale column c4 (0..3) of token-row r (0..127) inside a
// 512-byte scale atom.
__device__ __forceinline__ int atom_off(int r, int c4) { return 16 * (r & 31) + 4 * (r >> 5) + c4; }

// Scale code and 1/scale of a block with the given amax (>= 0).
__device__ __forceinline__ uint32_t block_scale(float amax, float &rcp) {
    const uint32_t sc = cvt_e4m3(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_value(sc);
    rcp = (s == 0.0f) ? 0.0f : __frcp_rn(s);
    return sc;
}

__device__ __forceinline__ uint32_t codes8(const float (&x)[8], float r) {
    if (r == 0.0f) return 0u;  // scale 0: every code is 0 (+0)
    return cvt_e2m1x8(__fmul_rn(x[0], r), __fmul_rn(x[1], r), __fmul_rn(x[2], r), __fmul_rn(x[3], r),
                      __fmul_rn(x[4], r), __fmul_rn(x[5], r), __fmul_rn(x[6], r), __fmul_rn(x[7], r));
}

// One 128-token tile of Q or K (blocks of 16 along d).
template <int D, bool kSmooth>
__device__ __forceinline__ void qk_tile(const __nv_bfloat16 *__restrict__ src, int N, int tile,
                                        const float *__restrict__ mean, uint8_t *__restrict__ codes,
                                        uint8_t *__restrict__ sf) {
    constexpr int kVec = D / 8;  // 16-byte vectors per row
    constexpr int kIters = kTile * kVec / kThreads;
    const int tid = threadIdx.x;
    uint4 raw[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int hb = it * kThreads + tid;
        const int t = tile * kTile + hb / kVec;
        raw[it] = (t < N) ? ld_stream_v4(src + static_cast<size_t>(t) * D + (hb % kVec) * 8)
                          : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int hb = it * kThreads + tid;
        const int row = hb / kVec;
        const int v = hb % kVec;
        const int t = tile * kTile + row;
        float x[8];
        bf16x8(raw[it], x);
        if (kSmooth && t < N) {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = __fsub_rn(x[i], mean[v * 8 + i]);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        float r;
        const uint32_t sc = block_scale(amax, r);
        *reinterpret_cast<uint32_t *>(codes + static_cast<size_t>(t) * (D / 2) + v * 4) = codes8(x, r);
        if ((v & 1) == 0) {
            const int blk = v >> 1;
            sf[(static_cast<size_t>(tile) * (D / 64) + (blk >> 2)) * 512 + atom_off(row, blk & 3)] =
                static_cast<uint8_t>(sc);
        }
    }
}

// Quantize the 16 tokens (16*tb .. 16*tb+15 of this tile) of channel c.
template <int D>
__device__ __forceinline__ void store_vblock(const float (&x)[16], int c, int tile, int tb, int Np,
                                             uint8_t *__restrict__ vt, uint8_t *__restrict__ vsf) {
    float amax = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(x[k]));
    float r;
    const uint32_t sc = block_scale(amax, r);
    const float lo[8] = {x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]};
    const float hi[8] = {x[8], x[9], x[10], x[11], x[12], x[13], x[14], x[15]};
    uint2 w;
    w.x = codes8(lo, r);
    w.y = codes8(hi, r);
    *reinterpret_cast<uint2 *>(vt + static_cast<size_t>(c) * (Np / 2) + tile * 64 + tb * 8) = w;
    const size_t g = static_cast<size_t>(tile * 2 + (tb >> 2)) * 512;
    vsf[g + 16 * (c & 31) + 4 * (c >> 5) + (tb & 3)] = static_cast<uint8_t>(sc);
    if (D < 128) {  // padding channels of the 128-row scale atom
        const int cz = c + D;
        vsf[g + 16 * (cz & 31) + 4 * (cz >> 5) + (tb & 3)] = 0;
    }
}

// One 128-token tile of V, quantized transposed (blocks of 16 tokens per
// channel).  stage: 128 x D bf16 in shared memory.
template <int D>
__device__ __forceinline__ void v_tile(const __nv_bfloat16 *__restrict__ src, int N, int Np, int tile,
                                       uint8_t *__restrict__ vt, uint8_t *__restrict__ vsf, uint32_t *stage) {
    constexpr int kVec = D / 8;
    constexpr int kWords = D / 2;  // 32-bit words per staged row
    constexpr int kIters = kTile * kVec / kThreads;
    const int tid = threadIdx.x;
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int hb = it * kThreads + tid;
        const int row = hb / kVec;
        const int v = hb % kVec;
        const int t = tile * kTile + row;
        const uint4 val = (t < N) ? ld_stream_v4(src + static_cast<size_t>(t) * D + v * 8) : make_uint4(0u, 0u, 0u, 0u);
        const int vs = v ^ ((row >> 4) & 7);
        *reinterpret_cast<uint4 *>(stage + row * kWords + vs * 4) = val;
    }
    __syncthreads();
    constexpr int kUnits = (D / 2) * 8;  // (channel pair, 16-token block)
    for (int u = tid; u < kUnits; u += kThreads) {
        const int tb = u & 7;
        const int cp = u >> 3;
        float x0[16], x1[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int row = tb * 16 + k;
            const uint32_t w = stage[row * kWords + (((cp >> 2) ^ tb) << 2) + (cp & 3)];
            x0[k] = __uint_as_float(w << 16);
            x1[k] = __uint_as_float(w & 0xFFFF0000u);
        }
        store_vblock<D>(x0, 2 * cp, tile, tb, Np, vt, vsf);
        store_vblock<D>(x1, 2 * cp + 1, tile, tb, Np, vt, vsf);
    }
}

// fp64 partial sums of K over one 512-token chunk.
template <int D>
__device__ __forceinline__ void k_partial(const __nv_bfloat16 *__restrict__ src, int N, int chunk, int chunk_len,
                                          double *__restrict__ part, double *red) {
    constexpr int kVec = D / 8;
    constexpr int kRows = kThreads / kVec;  // rows covered per step
    const int tid = threadIdx.x;
    const int v = tid % kVec;
    const int r0 = tid / kVec;
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    const int t0 = chunk * chunk_len;
    const int t1 = min(N, t0 + chunk_len);
    constexpr int kBatch = 8;
    for (int tb = t0 + r0; tb < t1; tb += kRows * kBatch) {
        uint4 raw[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int t = tb + b * kRows;
            raw[b] = (t < t1) ? ld_stream_v4(src + static_cast<size_t>(t) * D + v * 8) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            float x[8];
            bf16x8(raw[b], x);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(x[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[r0 * D + v * 8 + i] = acc[i];
    __syncthreads();
    for (int c = tid; c < D; c += kThreads) {
        double s = 0.0;
        for (int r = 0; r < kRows; ++r) s += red[r * D + c];
        part[static_cast<size_t>(chunk) * D + c] = s;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 4) quant_qv_ksum_kernel(QuantParams p) {
    __shared__ __align__(16) uint8_t smem[kTile * D * 2];
    const int bh = blockIdx.y;
    const int x = blockIdx.x;
    const size_t in_off = static_cast<size_t>(bh) * p.N * D;
    if (blockIdx.z == 0) {  // Q
        qk_tile<D, false>(p.q + in_off, p.N, x, nullptr,
                          p.q_fp4 + static_cast<size_t>(bh) * p.Np * (D / 2),
                          p.q_sf + static_cast<size_t>(bh) * p.Np * (D / 16));
    } else if (blockIdx.z == 1) {  // V
        v_tile<D>(p.v + in_off, p.N, p.Np, x, p.vt_fp4 + static_cast<size_t>(bh) * D * (p.Np / 2),
                  p.vt_sf + static_cast<size_t>(bh) * p.Np * 8, reinterpret_cast<uint32_t *>(smem));
    } else {  // K partial sums
        if (x >= p.nchunk) return;
        k_partial<D>(p.k + in_off, p.N, x, p.chunk, p.part + static_cast<size_t>(bh) * p.nchunk * D,
                     reinterpret_cast<double *>(smem));
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads) quant_k_kernel(QuantParams p) {
    __shared__ float mean[D];
    const int bh = blockIdx.y;
    // mean of K over its N tokens: partial sums added in chunk order (fp64),
    // one division, one rounding to fp32; tile 0 also stores it
    for (int c = threadIdx.x; c < D; c += kThreads) {
        const double *part = p.part + static_cast<size_t>(bh) * p.nchunk * D + c;
        double s = 0.0;
        for (int ch = 0; ch < p.nchunk; ++ch) s += part[static_cast<size_t>(ch) * D];
        const float mu = __double2float_rn(s / static_cast<double>(p.N));
        mean[c] = mu;
        if (blockIdx.x == 0) p.k_mean[static_cast<size_t>(bh) * D + c] = mu;
    }
    __syncthreads();
    qk_tile<D, true>(p.k + static_cast<size_t>(bh) * p.N * D, p.N, blockIdx.x, mean,
                     p.k_fp4 + static_cast<size_t>(bh) * p.Np * (D / 2),
                     p.k_sf + static_cast<size_t>(bh) * p.Np * (D / 16));
}

template <int D>
cudaError_t launch_quant_d(const QuantParams &p, cudaStream_t stream) {
    const int ntile = p.Np / kTile;
    quant_qv_ksum_kernel<D><<<dim3(ntile, p.BH, 3), kThreads, 0, stream>>>(p);
    quant_k_kernel<D><<<dim3(ntile, p.BH, 1), kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

inline cudaError_t launch_quant(const QuantParams &p, int d, cudaStream_t stream) {
    return d == 128 ? launch_quant_d<128>(p, stream) : launch_quant_d<64>(p, stream);
}

}  // namespace sa3
