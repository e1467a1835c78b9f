// quant.cuh -- K smoothing and FP4 microscaling of Q, K and V.
//
// Method: "SageAttention: Accurate 8-Bit Attention for Plug-and-play
// Inference Acceleration" (summary, section "Approach") smooths K by
// subtracting its mean over tokens; "SageAttention3: Microscaling FP4
// Attention ..." (abstract) runs attention on microscaled FP4 operands:
// E2M1 codes with one E4M3 scale per 16 elements.  The exact recipe of one
// block (x_0..x_15):  s = E4M3_RN_sat(amax/6), r = 1/s, code_i =
// E2M1_RN_sat(x_i * r), all zero if s == 0 -- see include/sa3.h.
//
// HBM-bound streaming work in two launches on the caller's stream, both
// made of persistent CTAs (two per SM) that stream 128-token bf16 tiles
// through a ring of shared-memory buffers filled by 3-D TMA loads (64
// channels x 128 tokens per box, 128-byte swizzle, rows past N zero-filled
// by the copy engine):
//   A  each CTA takes a balanced static share of the Q and V tiles and then
//      of the K chunks (fp64 column sums of K over at most 16 token chunks
//      per (b, h)); K comes last so that it is still in L2 for B;
//   B  K tiles, launched as a programmatic dependent of A: each CTA starts
//      its first K loads, waits for A, forms the mean of each (b, h) it
//      meets from the chunk sums (in chunk order, fp64), then smooths and
//      quantizes its contiguous range of tiles.
// Thread layouts (256 threads per CTA), all conflict-free on the swizzled
// tiles: Q/K tiles -- a thread owns D/32 consecutive 16-element blocks of
// one token row, the 8 threads of each shared-memory phase on 8 different
// rows; V tiles (quantized transposed, 16 tokens per block) -- a
// thread owns a pair of channels over D/64 consecutive 16-token blocks,
// warps reading 32 consecutive channel pairs of one token row at a time;
// K sums -- a thread owns 8 channels of every 16th (D=128) or 32nd (D=64)
// row and the warps' fp64 sums are added in a fixed order.
#pragma once

#include "sa3_internal.h"
#include "sm100.cuh"

namespace sa3 {
namespace quant {

constexpr int kTile = 128;      // tokens per tile
constexpr int kThreads = 256;   // threads per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 3;      // tile buffers per CTA
constexpr int kCtasPerSm = 2;
constexpr int kMaxChunks = 16;  // sa3_kmean_chunk keeps the chunk count at or below this
constexpr int kBoxCh = 64;      // channels per TMA box (128 bytes of bf16)

template <int D>
struct QCfg {
    static constexpr int kBoxBytes = kTile * kBoxCh * 2;  // 16 KB
    static constexpr int kTileBytes = kTile * D * 2;      // D/64 boxes
    static constexpr int oStage = 0;
    static constexpr int oRed = kStages * kTileBytes;     // fp64 K sums: one row of D per warp
    static constexpr int oLut = oRed + kWarps * D * 8;    // 256 floats: 1 / E4M3 value
    static constexpr int oMean = oLut + 256 * 4;          // -mean of K, D floats
    static constexpr int oBar = oMean + D * 4;            // kStages full barriers + abort flag
    static constexpr int kSmemBytes = oBar + kStages * 8 + 16 + 1024;  // + alignment slack
};

// Byte offset of bf16 element (row, ch) inside a staged tile: box ch/64,
// 128-byte rows, 16-byte chunk index XOR (row % 8) (128-byte swizzle).
__device__ __forceinline__ int tile_off(int row, int ch) {
    return (ch >> 6) * (kTile * kBoxCh * 2) + row * 128 + ((((ch & 63) >> 3) ^ (row & 7)) << 4) + (ch & 7) * 2;
}

// Byte offset of scale column c4 (0..3) of token-row r (0..127) inside a
// 512-byte scale atom.
__device__ __forceinline__ int atom_off(int r, int c4) { return 16 * (r & 31) + 4 * (r >> 5) + c4; }


// Exact 1/s for every E4M3 scale code s (0 for the zero code and NaN codes,
// which the saturating conversion never produces).
__device__ __forceinline__ void fill_rcp_lut(float *lut) {
    for (int i = threadIdx.x; i < 256; i += kThreads) {
        const float v = e4m3_value(static_cast<uint32_t>(i));
        lut[i] = (v == 0.0f || v != v) ? 0.0f : __frcp_rn(v);
    }
}

// Token row and channel half of thread t (0..255) in a Q/K tile: eight
// consecutive threads take one channel half of eight consecutive rows, so
// their 16-byte shared-memory reads fall in eight different bank groups.
__host__ __device__ __forceinline__ int qk_row(int t) { return (t & 7) | ((t >> 4) << 3); }
__host__ __device__ __forceinline__ int qk_part(int t) { return (t >> 3) & 1; }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// fp32(x / 6) without a division, after Brisebarre, Muller and Raina,
// "Accelerating Correctly Rounded Floating-Point Division when the Divisor
// Is Known in Advance" (IEEE Trans. Computers 53(8), 2004): with
// zh = RN(1/6) and zl = RN(1/6 - zh), RN(zh*x + RN(zl*x)) is the correctly
// rounded quotient for every fp32 x >= 2^-122.  Below that, zl*x
// underflows and the result may be off, but it and x / 6 both lie far
// under 2^-10, half the smallest E4M3 step, so the scale code is 0 either
// way; x = inf is clamped to the largest float, whose quotient saturates
// the scale just as inf / 6 does.  tests/div6_check.c checks all of this
// for every non-negative fp32 x.
__host__ __device__ __forceinline__ float div6(float x) {
    x = fminf(x, 0x1.fffffep127f);
    return fmaf(x, 0x1.555556p-3f, x * -0x1.555556p-28f);
}

// Scale code of a block: E4M3_RN_sat(fp32(amax / 6)).
__device__ __forceinline__ uint32_t scale_code(float amax) { return cvt_e4m3(div6(amax)); }

// E2M1 codes of 16 values times r (fp32 products, rounded once each).
__device__ __forceinline__ uint2 codes16(const uint64_t (&x2)[8], float r) {
    if (r == 0.0f) return make_uint2(0u, 0u);  // scale 0: every code is 0 (+0)
    const uint64_t rr = pack2(r, r);
    float y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t v = mul2(x2[i], rr);
        y[2 * i] = lo2(v);
        y[2 * i + 1] = hi2(v);
    }
    return make_uint2(cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]),
                      cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]));
}

// max(0, |x_0|, ..., |x_15|), NaNs ignored, as a tree (max is exact, so
// any order gives the same value).
__device__ __forceinline__ float amax16(const uint64_t (&x2)[8]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(fabsf(lo2(x2[i])), fabsf(hi2(x2[i])));
#pragma unroll
    for (int w = 4; w > 0; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
    }
    return fmaxf(m[0], 0.0f);
}

// ---------------------------------------------------------------- tiles
// Quantizes the D/32 consecutive 16-element blocks of token row `row`,
// channel half `part`, of a staged tile along d: E2M1 codes into cw (two
// words per block), the blocks' scale codes packed one byte each into the
// return value.  smooth: add neg_mean (-mean of K per channel; negation is
// exact, so x + (-mean) is the fp32 subtraction x - mean) first.  The
// attention kernel's Q-on-load path calls this too, so both produce the
// same codes by construction.
template <int D>
__device__ __forceinline__ uint32_t row_part_codes(const uint8_t *__restrict__ stage, int row, int part, bool smooth,
                                                   const float *__restrict__ neg_mean,
                                                   const float *__restrict__ rcp_lut, uint32_t (&cw)[D / 16]) {
    constexpr int kBpt = D / 32;
    uint32_t scw = 0;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) {
        const int ch0 = (part * kBpt + i) * 16;
        const uint4 a = *reinterpret_cast<const uint4 *>(stage + tile_off(row, ch0));
        const uint4 b = *reinterpret_cast<const uint4 *>(stage + tile_off(row, ch0 + 8));
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint64_t x2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x2[e] = pack2(bf16_lo(w[e]), bf16_hi(w[e]));
        if (smooth) {
            const float4 *nm = reinterpret_cast<const float4 *>(neg_mean + ch0);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 m4 = nm[e];
                x2[2 * e] = add2(x2[2 * e], pack2(m4.x, m4.y));
                x2[2 * e + 1] = add2(x2[2 * e + 1], pack2(m4.z, m4.w));
            }
        }
        const uint32_t sc = scale_code(amax16(x2));
        const uint2 c = codes16(x2, rcp_lut[sc]);
        cw[2 * i] = c.x;
        cw[2 * i + 1] = c.y;
        scw |= sc << (8 * i);
    }
    return scw;
}

// One staged 128-token tile of Q or K, quantized along d.  neg_mean: -mean
// of K per channel (smoothing) or nullptr for Q.  Rows past N arrive as
// zeros and get code 0 and scale 0.
template <int D, bool kSmooth>
__device__ __forceinline__ void qk_tile(const uint8_t *__restrict__ stage, int N, int tile,
                                        const float *__restrict__ neg_mean, const float *__restrict__ rcp_lut,
                                        uint8_t *__restrict__ codes, uint8_t *__restrict__ sf, bool st32) {
    constexpr int kBpt = D / 32;  // 16-element blocks per thread (4 or 2), consecutive along d
    const int row = qk_row(static_cast<int>(threadIdx.x));
    const int part = qk_part(static_cast<int>(threadIdx.x));
    const int t = tile * kTile + row;
    uint32_t cw[2 * kBpt];
    const uint32_t scw = row_part_codes<D>(stage, row, part, kSmooth && t < N, neg_mean, rcp_lut, cw);
    uint8_t *dst = codes + static_cast<size_t>(t) * (D / 2) + part * (kBpt * 8);
    if constexpr (kBpt == 4) {
        if (st32) {
            st_global_v8(dst, cw);
        } else {
            reinterpret_cast<uint4 *>(dst)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            reinterpret_cast<uint4 *>(dst)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
        }
        // blocks 4*part .. 4*part+3 are the four columns of atom `part`
        *reinterpret_cast<uint32_t *>(sf + static_cast<size_t>(tile * 2 + part) * 512 + atom_off(row, 0)) = scw;
    } else {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        // blocks 2*part, 2*part+1: columns 2*part, 2*part+1 of the tile's atom
        *reinterpret_cast<uint16_t *>(sf + static_cast<size_t>(tile) * 512 + atom_off(row, 2 * part)) =
            static_cast<uint16_t>(scw);
    }
}

// One staged 128-token tile of V, quantized transposed: blocks of 16 tokens
// per channel.  Thread: channel pair (2cp, 2cp+1), 16-token blocks
// g*D/64 .. g*D/64 + D/64 - 1.  kSmooth: -mean of V per channel is added to
// tokens t < N (the fp32 subtraction V - mean, as for K); padding tokens
// stay 0.
template <int D, bool kSmooth>
__device__ __forceinline__ void v_tile(const uint8_t *__restrict__ stage, int N, int Np, int tile,
                                       const float *__restrict__ neg_mean, const float *__restrict__ rcp_lut,
                                       uint8_t *__restrict__ vt, uint8_t *__restrict__ vsf) {
    constexpr int kPairs = D / 2;
    constexpr int kTbpt = D / 64;  // 16-token blocks per thread (2 or 1)
    const int cp = static_cast<int>(threadIdx.x) % kPairs;
    const int g = static_cast<int>(threadIdx.x) / kPairs;
    float nm0 = 0.0f, nm1 = 0.0f;
    if constexpr (kSmooth) {
        nm0 = neg_mean[2 * cp];
        nm1 = neg_mean[2 * cp + 1];
    }
    uint32_t c0[2 * kTbpt], c1[2 * kTbpt];
    uint32_t s0 = 0, s1 = 0;
#pragma unroll
    for (int i = 0; i < kTbpt; ++i) {
        const int tb = g * kTbpt + i;
        uint64_t x0[8], x1[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
            const int r = tb * 16 + k;
            const uint32_t w0 = *reinterpret_cast<const uint32_t *>(stage + tile_off(r, 2 * cp));
            const uint32_t w1 = *reinterpret_cast<const uint32_t *>(stage + tile_off(r + 1, 2 * cp));
            x0[k / 2] = pack2(bf16_lo(w0), bf16_lo(w1));
            x1[k / 2] = pack2(bf16_hi(w0), bf16_hi(w1));
            if constexpr (kSmooth) {
                const int t = tile * kTile + r;  // tokens t, t+1 (channel pairs 2cp, 2cp+1)
                x0[k / 2] = add2(x0[k / 2], pack2(t < N ? nm0 : 0.0f, t + 1 < N ? nm0 : 0.0f));
                x1[k / 2] = add2(x1[k / 2], pack2(t < N ? nm1 : 0.0f, t + 1 < N ? nm1 : 0.0f));
            }
        }
        const uint32_t sc0 = scale_code(amax16(x0));
        const uint32_t sc1 = scale_code(amax16(x1));
        const uint2 q0 = codes16(x0, rcp_lut[sc0]);
        const uint2 q1 = codes16(x1, rcp_lut[sc1]);
        c0[2 * i] = q0.x;
        c0[2 * i + 1] = q0.y;
        c1[2 * i] = q1.x;
        c1[2 * i + 1] = q1.y;
        s0 |= sc0 << (8 * i);
        s1 |= sc1 << (8 * i);
    }
    const int c = 2 * cp;
    uint8_t *row0 = vt + static_cast<size_t>(c) * (Np / 2) + tile * 64 + g * (kTbpt * 8);
    uint8_t *row1 = row0 + Np / 2;
    const int tb0 = g * kTbpt;
    uint8_t *atom = vsf + static_cast<size_t>(tile * 2 + (tb0 >> 2)) * 512;
    if constexpr (kTbpt == 2) {
        *reinterpret_cast<uint4 *>(row0) = make_uint4(c0[0], c0[1], c0[2], c0[3]);
        *reinterpret_cast<uint4 *>(row1) = make_uint4(c1[0], c1[1], c1[2], c1[3]);
        *reinterpret_cast<uint16_t *>(atom + atom_off(c, tb0 & 3)) = static_cast<uint16_t>(s0);
        *reinterpret_cast<uint16_t *>(atom + atom_off(c + 1, tb0 & 3)) = static_cast<uint16_t>(s1);
    } else {
        *reinterpret_cast<uint2 *>(row0) = make_uint2(c0[0], c0[1]);
        *reinterpret_cast<uint2 *>(row1) = make_uint2(c1[0], c1[1]);
        atom[atom_off(c, tb0 & 3)] = static_cast<uint8_t>(s0);
        atom[atom_off(c + 1, tb0 & 3)] = static_cast<uint8_t>(s1);
        // channels D .. 127 of the 128-row scale atom are padding (scale 0)
        atom[atom_off(c + D, tb0 & 3)] = 0;
        atom[atom_off(c + 1 + D, tb0 & 3)] = 0;
    }
}

// ------------------------------------------------- 8-bit variant tiles
// One staged 128-token tile of Q or K as INT8 with one scale for the whole
// tile ("SageAttention" summary, "Approach"; per-block scales):
// s = fp32(amax / 127), r = fp32(1 / s), code = clamp(rn_even(fp32(x r)),
// +-127).  Thread: token row qk_row(t), channel half qk_part(t).  red: 8 floats of
// shared scratch.  Returns nothing; thread 0 stores the scale.
template <int D, bool kSmooth>
__device__ __forceinline__ void qk_tile_i8(const uint8_t *__restrict__ stage, int N, int tile,
                                           const float *__restrict__ neg_mean, int8_t *__restrict__ codes,
                                           float *__restrict__ scale_out, float *red, bool st32) {
    constexpr int kCh = D / 2;  // channels per thread
    const int row = qk_row(static_cast<int>(threadIdx.x));
    const int part = qk_part(static_cast<int>(threadIdx.x));
    const int t = tile * kTile + row;
    float x[kCh];
    float amax = 0.0f;
#pragma unroll
    for (int c8 = 0; c8 < kCh / 8; ++c8) {
        const int ch0 = part * kCh + c8 * 8;
        const uint4 w = *reinterpret_cast<const uint4 *>(stage + tile_off(row, ch0));
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[c8 * 8 + 2 * e] = bf16_lo(u[e]);
            x[c8 * 8 + 2 * e + 1] = bf16_hi(u[e]);
        }
        if (kSmooth && t < N) {
#pragma unroll
            for (int e = 0; e < 8; ++e) x[c8 * 8 + e] = __fadd_rn(x[c8 * 8 + e], neg_mean[ch0 + e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[c8 * 8 + e]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    float a = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) a = fmaxf(a, red[w]);
    const float s = __fdiv_rn(a, 127.0f);
    const float r = s == 0.0f ? 0.0f : __frcp_rn(s);
    uint32_t pk[kCh / 4];
#pragma unroll
    for (int i = 0; i < kCh / 4; ++i) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int c = __float2int_rn(__fmul_rn(x[4 * i + e], r));  // round half to even
            c = c > 127 ? 127 : (c < -127 ? -127 : c);
            word |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * e);
        }
        pk[i] = word;
    }
    int8_t *dst = codes + static_cast<size_t>(t) * D + part * kCh;
    if (st32) {
#pragma unroll
        for (int i = 0; i < kCh / 32; ++i) {
            const uint32_t w[8] = {pk[8 * i], pk[8 * i + 1], pk[8 * i + 2], pk[8 * i + 3],
                                   pk[8 * i + 4], pk[8 * i + 5], pk[8 * i + 6], pk[8 * i + 7]};
            st_global_v8(dst + 32 * i, w);
        }
    } else {
#pragma unroll
        for (int i = 0; i < kCh / 16; ++i)
            reinterpret_cast<uint4 *>(dst)[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
    if (threadIdx.x == 0) scale_out[tile] = s;
    // red is rewritten by the next Q or K tile only after the caller's
    // __syncthreads that follows every tile
}

// One staged 128-token tile of V as FP16 (round to nearest even), stored
// transposed: vt [d][Np] halves.  Thread: channel pair (2cp, 2cp+1),
// 16-token blocks g*D/64 .. g*D/64 + D/64 - 1, one 32-byte row piece per
// channel and block.
template <int D>
__device__ __forceinline__ void v_tile_f16(const uint8_t *__restrict__ stage, int Np, int tile,
                                           uint8_t *__restrict__ vt, bool st32) {
    constexpr int kPairs = D / 2;
    constexpr int kTbpt = D / 64;
    const int cp = static_cast<int>(threadIdx.x) % kPairs;
    const int g = static_cast<int>(threadIdx.x) / kPairs;
#pragma unroll
    for (int i = 0; i < kTbpt; ++i) {
        const int tb = g * kTbpt + i;
        uint32_t h0[8], h1[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
            const int r = tb * 16 + k;
            const uint32_t w0 = *reinterpret_cast<const uint32_t *>(stage + tile_off(r, 2 * cp));
            const uint32_t w1 = *reinterpret_cast<const uint32_t *>(stage + tile_off(r + 1, 2 * cp));
            const __half2 a = __floats2half2_rn(bf16_lo(w0), bf16_lo(w1));  // channel 2cp, tokens r, r+1
            const __half2 b = __floats2half2_rn(bf16_hi(w0), bf16_hi(w1));  // channel 2cp+1
            h0[k / 2] = *reinterpret_cast<const uint32_t *>(&a);
            h1[k / 2] = *reinterpret_cast<const uint32_t *>(&b);
        }
        uint8_t *r0 = vt + (static_cast<size_t>(2 * cp) * Np + tile * kTile + tb * 16) * 2;
        uint8_t *r1 = r0 + static_cast<size_t>(Np) * 2;
        if (st32) {
            st_global_v8(r0, h0);
            st_global_v8(r1, h1);
        } else {
            reinterpret_cast<uint4 *>(r0)[0] = make_uint4(h0[0], h0[1], h0[2], h0[3]);
            reinterpret_cast<uint4 *>(r0)[1] = make_uint4(h0[4], h0[5], h0[6], h0[7]);
            reinterpret_cast<uint4 *>(r1)[0] = make_uint4(h1[0], h1[1], h1[2], h1[3]);
            reinterpret_cast<uint4 *>(r1)[1] = make_uint4(h1[4], h1[5], h1[6], h1[7]);
        }
    }
}

// fp64 column sums of one staged K tile into this thread's accumulators:
// channels 8v .. 8v+7 of rows r0, r0 + kRowStep, ...
template <int D>
__device__ __forceinline__ void ksum_tile(const uint8_t *__restrict__ stage, double (&acc)[8]) {
    constexpr int kVec = D / 8;
    constexpr int kRowStep = kThreads / kVec;
    const int v = static_cast<int>(threadIdx.x) % kVec;
    const int r0 = static_cast<int>(threadIdx.x) / kVec;
#pragma unroll
    for (int r = r0; r < kTile; r += kRowStep) {
        const uint4 w = *reinterpret_cast<const uint4 *>(stage + tile_off(r, v * 8));
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[2 * e] += static_cast<double>(bf16_lo(u[e]));
            acc[2 * e + 1] += static_cast<double>(bf16_hi(u[e]));
        }
    }
}

// Adds every thread's accumulators of the current chunk (warp shuffles over
// the lanes holding the same channels, then the warps in order) and writes
// the chunk's D sums; clears the accumulators.  Called by all threads.
template <int D>
__device__ __forceinline__ void ksum_flush(double (&acc)[8], double *red, double *__restrict__ out) {
    constexpr int kVec = D / 8;
    const int warp = static_cast<int>(threadIdx.x) >> 5;
    const int lane = static_cast<int>(threadIdx.x) & 31;
#pragma unroll
    for (int off = kVec; off < 32; off <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    }
    if (lane < kVec) {
#pragma unroll
        for (int i = 0; i < 8; ++i) red[warp * D + lane * 8 + i] = acc[i];
    }
    __syncthreads();
    for (int c = static_cast<int>(threadIdx.x); c < D; c += kThreads) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w * D + c];
        out[c] = s;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
}

// ------------------------------------------------------------- schedule
// Work of the first launch for CTA g of G: a contiguous range of the Q and
// V tiles (Q tiles of every (b, h) first, then V; Q and V may have different
// token counts), then the column-sum chunks g, g+G, g+2G, ... one tile at a
// time: K's chunks, then (V smoothing) V's, whose tiles then go to the
// second launch instead.  The Q/V ranges are sized so that every CTA ends
// up with about the same number of tiles: CTAs holding one chunk more (the
// first nK % G) take tpc fewer Q/V tiles.
struct TileJob {
    int kind;  // 0 = Q, 1 = V, 2 = K column sums, 3 = V column sums
    int bh;
    int tile;
    int chunk;      // sums: chunk of the tile
    bool last;      // sums: last tile of its chunk
};

struct SchedA {
    int ntile_q, ntile, nchunk, tpc, nqk, nsum;  // nqk = BH * ntile_q (Q tiles; V tiles follow)
    int j, je;                    // Q/V tiles [j, je)
    int ki, nK, G;                // next chunk item, items, stride
    int kkind, kbh, kch, kt, kt_end;  // current chunk (2 = K, 3 = V) and its tiles [kt, kt_end)

    __host__ __device__ void init(int BH, int ntile_q_, int ntile_, int nchunk_, int tpc_, int g, int G_,
                                  bool vsmooth = false) {
        ntile_q = ntile_q_;
        ntile = ntile_;
        nchunk = nchunk_;
        tpc = tpc_;
        nqk = BH * ntile_q;
        G = G_;
        nsum = BH * nchunk;
        nK = nsum * (vsmooth ? 2 : 1);
        const int nqv = nqk + (vsmooth ? 0 : BH * ntile);
        const int r = nK % G;
        long long q_hi = (static_cast<long long>(nqv) + static_cast<long long>(r) * tpc + G - 1) / G;
        long long q_lo = q_hi - tpc;
        if (q_lo < 0) {
            q_lo = 0;
            q_hi = (nqv + (G - r) - 1) / (G - r);
        }
        const long long pre = g < r ? g * q_lo : r * q_lo + static_cast<long long>(g - r) * q_hi;
        const long long cnt = g < r ? q_lo : q_hi;
        j = static_cast<int>(pre < nqv ? pre : nqv);
        je = static_cast<int>(pre + cnt < nqv ? pre + cnt : nqv);
        ki = g;
        kt = kt_end = 0;
        kkind = 2;
        kbh = kch = 0;
    }
    __host__ __device__ bool next(TileJob &t) {
        if (j < je) {
            const int kind = j < nqk ? 0 : 1;
            const int jj = kind ? j - nqk : j;
            const int nt = kind ? ntile : ntile_q;
            t.kind = kind;
            t.bh = jj / nt;
            t.tile = jj % nt;
            t.chunk = 0;
            t.last = false;
            ++j;
            return true;
        }
        if (kt >= kt_end) {
            if (ki >= nK) return false;
            kkind = ki < nsum ? 2 : 3;
            const int kk = ki < nsum ? ki : ki - nsum;
            kbh = kk / nchunk;
            kch = kk % nchunk;
            kt = kch * tpc;
            kt_end = kt + tpc < ntile ? kt + tpc : ntile;
            ki += G;
        }
        t.kind = kkind;
        t.bh = kbh;
        t.tile = kt;
        t.chunk = kch;
        t.last = kt + 1 == kt_end;
        ++kt;
        return true;
    }
};

// ---------------------------------------------------------------- ring
// kStages tile buffers, each filled by D/64 TMA boxes and one full barrier.
template <int D>
__device__ __forceinline__ void ring_issue(uint8_t *stage, uint64_t *full, const CUtensorMap *map, int bh,
                                           int tile, uint64_t policy) {
    mbar_arrive_expect_tx(full, QCfg<D>::kTileBytes);
#pragma unroll
    for (int b = 0; b < D / 64; ++b)
        tma_load_3d_hint(stage + b * QCfg<D>::kBoxBytes, map, b * kBoxCh, tile * kTile, bh, full, policy);
}

// Thread 0, after a failed wait: let every copy still in flight land
// (bounded, ignoring the abort flag) before the CTA exits.
__device__ __forceinline__ void ring_drain(uint64_t *full, int consumed, int issued) {
    for (int m = consumed; m < issued; ++m) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(full + m % kStages, (m / kStages) & 1)) {
            if (globaltimer() - t0 > kWaitLimitNs) {
                atomicOr(&g_sa3_status, 1u);
                return;
            }
        }
    }
}

struct SmemPtrs {
    uint8_t *base;
    uint64_t *full;
    volatile int *abort;
    float *lut;
    double *red;
    float *neg_mean;
};

template <int D>
__device__ __forceinline__ SmemPtrs smem_setup(uint8_t *raw) {
    using C = QCfg<D>;
    const uint32_t a = smem_u32(raw);
    SmemPtrs s;
    s.base = raw + (((a + 1023u) & ~1023u) - a);
    s.full = reinterpret_cast<uint64_t *>(s.base + C::oBar);
    s.abort = reinterpret_cast<volatile int *>(s.full + kStages);
    s.lut = reinterpret_cast<float *>(s.base + C::oLut);
    s.red = reinterpret_cast<double *>(s.base + C::oRed);
    s.neg_mean = reinterpret_cast<float *>(s.base + C::oMean);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(s.full + i, 1);
        *s.abort = 0;
        fence_mbar_init();
    }
    fill_rcp_lut(s.lut);
    __syncthreads();
    return s;
}

// -------------------------------------------------------------- kernels
// First launch: Q and V tiles, then fp64 column sums of K per chunk.
// kI8: the 8-bit variant (INT8 Q, K with one scale per tile; FP16 V).
template <int D, bool kI8>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    quant_qvk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const QuantParams p) {
    extern __shared__ uint8_t smem_raw[];
    pdl_trigger();  // the second launch may start once every CTA of this one has
    const SmemPtrs sm = smem_setup<D>(smem_raw);
    SchedA prod, cons;
    prod.init(p.BH, p.Npq / kTile, p.Np / kTile, p.nchunk, p.chunk / kTile, static_cast<int>(blockIdx.x),
              static_cast<int>(gridDim.x), p.vsmooth != 0);
    cons = prod;
    const uint64_t pol_once = l2_policy_evict_first();
    const uint64_t pol_k = l2_policy_evict_normal();
    int issued = 0;
    auto issue_next = [&](int s) {
        TileJob t;
        if (!prod.next(t)) return;
        const CUtensorMap *m = t.kind == 0 ? &tm_q : (t.kind == 2 ? &tm_k : &tm_v);
        // column-summed K (and V) tiles are read again by the second launch
        ring_issue<D>(sm.base + s * QCfg<D>::kTileBytes, sm.full + s, m, t.bh, t.tile, t.kind >= 2 ? pol_k : pol_once);
        ++issued;
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) issue_next(s);
    }
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    int n = 0;
    bool ok = true;
    for (TileJob t; cons.next(t); ++n) {
        const int s = n % kStages;
        const bool got = mbar_wait(sm.full + s, (n / kStages) & 1, sm.abort);
        if (__syncthreads_or(!got)) {
            ok = false;
            break;
        }
        const uint8_t *st = sm.base + s * QCfg<D>::kTileBytes;
        if (t.kind == 0) {
            if constexpr (kI8)
                qk_tile_i8<D, false>(st, p.Nq, t.tile, nullptr,
                                     reinterpret_cast<int8_t *>(p.q_fp4) + static_cast<size_t>(t.bh) * p.Npq * D,
                                     p.q_scale + static_cast<size_t>(t.bh) * (p.Npq / kTile),
                                     reinterpret_cast<float *>(sm.red), p.st32 != 0);
            else
                qk_tile<D, false>(st, p.Nq, t.tile, nullptr, sm.lut,
                                  p.q_fp4 + static_cast<size_t>(t.bh) * p.Npq * (D / 2),
                                  p.q_sf + static_cast<size_t>(t.bh) * p.Npq * (D / 16), p.st32 != 0);
        } else if (t.kind == 1) {
            if constexpr (kI8)
                v_tile_f16<D>(st, p.Np, t.tile, p.vt_fp4 + static_cast<size_t>(t.bh) * D * p.Np * 2, p.st32 != 0);
            else
                v_tile<D, false>(st, p.N, p.Np, t.tile, nullptr, sm.lut,
                                 p.vt_fp4 + static_cast<size_t>(t.bh) * D * (p.Np / 2),
                                 p.vt_sf + static_cast<size_t>(t.bh) * p.Np * 8);
        } else {
            ksum_tile<D>(st, acc);
        }
        __syncthreads();  // stage s has been read by every thread
        if (t.kind >= 2 && t.last)
            ksum_flush<D>(acc, sm.red,
                          (t.kind == 2 ? p.part : p.vpart) + (static_cast<size_t>(t.bh) * p.nchunk + t.chunk) * D);
        if (threadIdx.x == 0) {
            fence_proxy_async_smem();
            issue_next(s);
        }
    }
    if (!ok && threadIdx.x == 0) ring_drain(sm.full, n, issued);
}

// Second launch: tiles [g*T/G, (g+1)*T/G) of the T = BH * ntile K tiles
// (then, with V smoothing, BH * ntile V tiles), each smoothed by the mean of
// its (b, h) and quantized.
template <int D, bool kI8>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    quant_k_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const QuantParams p) {
    extern __shared__ uint8_t smem_raw[];
    pdl_trigger();  // the attention launch behind this one may start its prologue
    const SmemPtrs sm = smem_setup<D>(smem_raw);
    const int ntile = p.Np / kTile;
    const long long nk = static_cast<long long>(p.BH) * ntile;
    const long long T = nk * (p.vsmooth ? 2 : 1);
    const int i0 = static_cast<int>(T * blockIdx.x / gridDim.x);
    const int i1 = static_cast<int>(T * (blockIdx.x + 1) / gridDim.x);
    const uint64_t pol = l2_policy_evict_first();
    auto issue = [&](int s, int idx) {
        const bool isv = idx >= nk;
        const int ii = isv ? idx - static_cast<int>(nk) : idx;
        ring_issue<D>(sm.base + s * QCfg<D>::kTileBytes, sm.full + s, isv ? &tm_v : &tm_k, ii / ntile, ii % ntile,
                      pol);
    };
    int issued = 0;
    // K and V are inputs of this launch, not outputs of the first one: their
    // loads may start before the wait below
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages && i0 + s < i1; ++s, ++issued) issue(s, i0 + s);
    }
    pdl_wait();
    int cur = -1;  // (kind, bh) whose mean is in neg_mean
    int n = 0;
    bool ok = true;
    for (; i0 + n < i1; ++n) {
        const int idx = i0 + n;
        const bool isv = idx >= nk;
        const int ii = isv ? idx - static_cast<int>(nk) : idx;
        const int bh = ii / ntile;
        const int tile = ii % ntile;
        if ((isv ? p.BH : 0) + bh != cur) {
            // mean over the N tokens: chunk sums added in chunk order (fp64),
            // one division, one rounding to fp32; the CTA holding tile 0 of
            // this (b, h) also stores it
            const double *part = (isv ? p.vpart : p.part) + static_cast<size_t>(bh) * p.nchunk * D;
            float *mean_out = isv ? p.v_mean : p.k_mean;
            for (int c = static_cast<int>(threadIdx.x); c < D; c += kThreads) {
                double v[kMaxChunks];
#pragma unroll
                for (int ch = 0; ch < kMaxChunks; ++ch)
                    v[ch] = ch < p.nchunk ? part[static_cast<size_t>(ch) * D + c] : 0.0;
                double sum = 0.0;
#pragma unroll
                for (int ch = 0; ch < kMaxChunks; ++ch)
                    if (ch < p.nchunk) sum += v[ch];
                const float mu = __double2float_rn(sum / static_cast<double>(p.N));
                sm.neg_mean[c] = -mu;
                if (tile == 0) mean_out[static_cast<size_t>(bh) * D + c] = mu;
            }
            __syncthreads();
            cur = (isv ? p.BH : 0) + bh;
        }
        const int s = n % kStages;
        const bool got = mbar_wait(sm.full + s, (n / kStages) & 1, sm.abort);
        if (__syncthreads_or(!got)) {
            ok = false;
            break;
        }
        const uint8_t *st = sm.base + s * QCfg<D>::kTileBytes;
        if constexpr (kI8) {
            qk_tile_i8<D, true>(st, p.N, tile, sm.neg_mean,
                                reinterpret_cast<int8_t *>(p.k_fp4) + static_cast<size_t>(bh) * p.Np * D,
                                p.k_scale + static_cast<size_t>(bh) * (p.Np / kTile), reinterpret_cast<float *>(sm.red),
                                p.st32 != 0);
        } else {
            if (isv)
                v_tile<D, true>(st, p.N, p.Np, tile, sm.neg_mean, sm.lut,
                                p.vt_fp4 + static_cast<size_t>(bh) * D * (p.Np / 2),
                                p.vt_sf + static_cast<size_t>(bh) * p.Np * 8);
            else
                qk_tile<D, true>(st, p.N, tile, sm.neg_mean, sm.lut, p.k_fp4 + static_cast<size_t>(bh) * p.Np * (D / 2),
                                 p.k_sf + static_cast<size_t>(bh) * p.Np * (D / 16), p.st32 != 0);
        }
        __syncthreads();  // stage s and neg_mean have been read by every thread
        if (threadIdx.x == 0 && i0 + n + kStages < i1) {
            fence_proxy_async_smem();
            issue(s, i0 + n + kStages);
            ++issued;
        }
    }
    if (!ok && threadIdx.x == 0) ring_drain(sm.full, n, issued);
}

template <int D, bool kI8>
cudaError_t launch_d(const QuantParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t stream) {
    using C = QCfg<D>;
    if (p.nchunk > kMaxChunks || p.chunk % kTile != 0) return cudaErrorInvalidValue;
    cudaError_t e = smem_attr_once<quant_qvk_kernel<D, kI8>>(C::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = smem_attr_once<quant_k_kernel<D, kI8>>(C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int nsm = sm_count();
    const long long ntile = p.Np / kTile;
    const long long work_a = static_cast<long long>(p.BH) * (p.Npq / kTile + (p.vsmooth ? 0 : ntile)) +
                             static_cast<long long>(p.BH) * p.nchunk * (p.vsmooth ? 2 : 1);
    const long long slots = static_cast<long long>(nsm) * kCtasPerSm;
    const int grid_a = static_cast<int>(work_a < slots ? work_a : slots);
    quant_qvk_kernel<D, kI8><<<grid_a, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long tiles_k = p.BH * ntile * (p.vsmooth ? 2 : 1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_k < slots ? tiles_k : slots));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quant_k_kernel<D, kI8>, tk, tv, p);
}

}  // namespace quant

// Two launches: Q/V tiles and K chunk sums, then smoothed K tiles.  tq, tk,
// tv: 3-D bf16 tensor maps {d, tokens, B*H} (Nq tokens for Q, N for K and V)
// with 64 x 128 boxes and 128-byte swizzle.
inline cudaError_t launch_quant(const QuantParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                                const CUtensorMap &tv, int d, cudaStream_t stream) {
    return d == 128 ? quant::launch_d<128, false>(p, tq, tk, tv, stream)
                    : quant::launch_d<64, false>(p, tq, tk, tv, stream);
}
// The 8-bit variant: INT8 Q, K (one fp32 scale per 128-token tile, K
// smoothed) and FP16 V^T, same schedule and launches.
inline cudaError_t launch_quant_i8(const QuantParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                                   const CUtensorMap &tv, int d, cudaStream_t stream) {
    return d == 128 ? quant::launch_d<128, true>(p, tq, tk, tv, stream)
                    : quant::launch_d<64, true>(p, tq, tk, tv, stream);
}

}  // namespace sa3
