// attn8.cuh -- the 8-bit variant of the attention forward for sm_100a.
//
// Method ("SageAttention: Accurate 8-Bit Attention for Plug-and-play
// Inference Acceleration", summary, "Approach"): Q and smoothed K in INT8
// with per-block scales, P and V in FP16.  Per 128-row Q tile and 128-key
// block j:
//   S = Q8 K8_j^T                       tcgen05.mma kind::i8, int32 in TMEM
//   t = S * f_j, f_j = fp32(fp32(s_q s_k,j) c)   (exact integer S)
//   m' = max(m, rowmax t), alpha = 2^(m - m'), P = 2^(t - m'),
//   l = alpha l + rowsum P, P16 = fp16(P)
//   O = alpha O + P16 V16_j             tcgen05.mma kind::f16, fp32 in TMEM
// and out = bf16(O / l); optionally lse = ln 2 (m + log2 l) per row, the
// softmax statistic that a backward pass of the training forward reuses.
//
// Same CTA organisation as the FP4 kernel (attn.cuh): two Q tiles per CTA,
// 16 softmax warps (two threads per row, exchanging partial row maxima),
// one TMA producer warp, one MMA-issuing warp; S in TMEM shared by the two
// tiles.  Differences: no block-scale factors (so no tcgen05.cp and no
// scale columns in TMEM); S is int32 and becomes fp32 exactly through the
// 1.5 * 2^23 bias trick (|S| <= 127 * 127 * 128 < 2^22); P is 16 bits, so a
// P tile is two 64-key 128-byte-swizzled atoms (32 KB) and a V^T tile two
// 64-key atoms of d rows; K and V^T have rings of their own (three K and
// two V^T slots at d = 128, four and three at d = 64).
#pragma once

#include "attn.cuh"

namespace sa3 {
namespace attn8 {

using attn::drain_wait;
using attn::ex2;
using attn::kBlk;
using attn::kSoftmaxWarps;
using attn::kThreads;
using attn::kWarpMma;
using attn::kWarpProducer;
using attn::max3f;
using attn::warp_wait;

template <int D>
struct Cfg {
    static constexpr int al(int x) { return (x + 1023) & ~1023; }
    // K and V^T in rings of their own: a K slot is free once both tiles'
    // S = Q K^T have run, a V^T slot only after both O += P V, so K can be
    // fetched further ahead than a shared K + V^T slot would allow
    static constexpr int kKStages = D == 128 ? 3 : 4;
    static constexpr int kVStages = D == 128 ? 2 : 3;
    // the producer issues K(j + kLead) before V^T(j): then both wait for
    // slots that the same MMA iteration frees
    static constexpr int kLead = kKStages + 1 - kVStages;
    static constexpr int kQBytes = kBlk * D;               // int8 Q or K tile: 128 rows x D bytes
    static constexpr int kAtomBytes = kBlk * 128;          // 128 rows x 64 halves
    static constexpr int kVAtomBytes = D * 128;            // D rows x 64 halves
    static constexpr int kVBytes = 2 * kVAtomBytes;        // V^T tile: D rows x 128 keys
    static constexpr int kPBytes = 2 * kAtomBytes;         // P tile: 128 rows x 128 keys
    static constexpr uint32_t kQKLayout = D == 128 ? 2u : 4u;  // 128B / 64B swizzle
    static constexpr uint32_t kQKSbo = 8 * D;
    // shared memory map, offsets from a 1024-byte aligned base
    static constexpr int oQ0 = 0;
    static constexpr int oQ1 = al(oQ0 + kQBytes);
    static constexpr int oK = al(oQ1 + kQBytes);          // K ring
    static constexpr int kKSlot = al(kQBytes);
    static constexpr int oV = oK + kKStages * kKSlot;     // V^T ring
    static constexpr int kVSlot = al(kVBytes);
    static constexpr int oP0 = oV + kVStages * kVSlot;
    static constexpr int oP1 = oP0 + kPBytes;
    static constexpr int oXch = oP1 + kPBytes;             // row maxima [2 parity][2 tiles][2 halves][128]
    static constexpr int oXl = oXch + 4096;                // row sums [2 tiles][2 halves][128]
    static constexpr int oBar = oXl + 2048;
    static constexpr int kSmemBytes = oBar + 256 + 1024;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    // TMEM columns
    static constexpr uint32_t tS = 0;
    static constexpr uint32_t tO0 = 128;
    static constexpr uint32_t tO1 = 128 + D;
    static constexpr uint32_t kTmemCols = 512;
};

constexpr int kMaxK = 4, kMaxV = 3;
enum : int {
    kBarQ = 0,
    kBarKFull = 1,                                  // kMaxK
    kBarKEmpty = kBarKFull + kMaxK,                 // kMaxK
    kBarVFull = kBarKEmpty + kMaxK,                 // kMaxV
    kBarVEmpty = kBarVFull + kMaxV,                 // kMaxV
    kBarSFull = kBarVEmpty + kMaxV,                 // 2
    kBarSEmpty = kBarSFull + 2,                     // 1
    kBarPFull = kBarSEmpty + 1,                     // 2
    kBarPvDone = kBarPFull + 2,                     // 2
    kBarDrain = kBarPvDone + 2,                     // 1
    kBarXch = kBarDrain + 1,                        // 8
    kBarCount = kBarXch + 8
};
static_assert(Cfg<128>::kKStages <= kMaxK && Cfg<64>::kKStages <= kMaxK && Cfg<128>::kVStages <= kMaxV &&
                  Cfg<64>::kVStages <= kMaxV,
              "ring barriers");
static_assert(kBarCount * 8 + 8 <= 256, "barrier area");

// Instruction descriptors (dense, K-major A and B, M = 128):
// kind::i8: signed int8 A and B, int32 D;  kind::f16: f16 A and B, f32 D.
__host__ __device__ constexpr uint32_t idesc_i8(int N) {
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (8u << 24);
}
__host__ __device__ constexpr uint32_t idesc_f16(int N) {
    return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (8u << 24);
}

__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// int32 (|x| < 2^22) -> fp32, exactly, on the integer and FMA pipes.
__device__ __forceinline__ float i2f_exact(uint32_t x) {
    return __fsub_rn(__uint_as_float(x + 0x4B400000u), 12582912.0f);
}

// Two fp32 -> packed fp16x2 (round to nearest even), low half from `lo`.
__device__ __forceinline__ uint32_t f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

template <int D, bool kCross>
__global__ void __launch_bounds__(kThreads, 1)
    attn8_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using C = Cfg<D>;
    constexpr int kK = C::kKStages;
    constexpr int kV = C::kVStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_s - raw_s);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + C::oBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kBarCount);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // work units as in the FP4 kernel: pairs of Q tiles, then single tiles
    const int nqt = p.Npq / kBlk;
    const int nkvt = p.Np / kBlk;
    const int off = kCross ? p.N - p.Nq : 0;
    const int u = static_cast<int>(blockIdx.x);
    const bool single = u >= p.pair_units;
    const int pu = single ? p.pair_units + (u - p.pair_units) / 2 : u;
    const int bh = pu % p.BH;
    const int rank = pu / p.BH;
    const int pair = p.causal ? p.npairs - 1 - rank : rank;
    const int tile0 = 2 * pair + (single ? ((u - p.pair_units) & 1) : 0);
    const int tile1 = tile0 + 1;
    if (tile0 >= nqt) return;
    const bool valid1 = !single && tile1 < nqt;
    auto n_blocks = [&](int tile) -> int {
        if (!p.causal) return nkvt;
        const int last = tile * kBlk + kBlk - 1 + off;
        const int nb = last < 0 ? 0 : last / kBlk + 1;
        return nb < nkvt ? nb : nkvt;
    };
    const int n0 = n_blocks(tile0);
    const int n1 = valid1 ? n_blocks(tile1) : 0;
    const int nmax = n0 > n1 ? n0 : n1;

    if (threadIdx.x == 0) {
        mbar_init(bars + kBarQ, 1);
        for (int s = 0; s < kK; ++s) {
            mbar_init(bars + kBarKFull + s, 1);
            mbar_init(bars + kBarKEmpty + s, 1);
        }
        for (int s = 0; s < kV; ++s) {
            mbar_init(bars + kBarVFull + s, 1);
            mbar_init(bars + kBarVEmpty + s, 1);
        }
        mbar_init(bars + kBarSFull + 0, 1);
        mbar_init(bars + kBarSFull + 1, 1);
        mbar_init(bars + kBarSEmpty, 256);
        mbar_init(bars + kBarPFull + 0, 256);
        mbar_init(bars + kBarPFull + 1, 256);
        mbar_init(bars + kBarPvDone + 0, 1);
        mbar_init(bars + kBarPvDone + 1, 1);
        mbar_init(bars + kBarDrain, 1);
        for (int x = 0; x < 8; ++x) mbar_init(bars + kBarXch + x, 64);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Launched as a programmatic dependent: everything above overlaps the
    // tail of the kernel before (the quantizer); every global read below
    // comes after it has completed
    pdl_wait();
    const uint32_t tmem = *tmem_slot;

    if (warp >= kWarpProducer) {
      if (warp == kWarpProducer) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            uint64_t *bq = bars + kBarQ;
            mbar_arrive_expect_tx(bq, (valid1 ? 2u : 1u) * C::kQBytes);
            tma_load_2d(base + C::oQ0, &tm_q, 0, bh * p.Npq + tile0 * kBlk, bq);
            if (valid1) tma_load_2d(base + C::oQ1, &tm_q, 0, bh * p.Npq + tile1 * kBlk, bq);
            // step t: K(t), then V^T(t - kLead); a wait for a slot depends
            // only on MMA iterations that the loads issued before it feed
            int k_issued = 0, v_issued = 0;
            for (int t = 0; t < nmax + C::kLead; ++t) {
                if (t < nmax) {
                    const int s = t % kK;
                    const int r = t / kK;
                    if (r > 0 && !mbar_wait(bars + kBarKEmpty + s, (r - 1) & 1, abort_flag)) break;
                    uint64_t *bf = bars + kBarKFull + s;
                    mbar_arrive_expect_tx(bf, C::kQBytes);
                    tma_load_2d(base + C::oK + s * C::kKSlot, &tm_k, 0, bh * p.Np + t * kBlk, bf);
                    k_issued = t + 1;
                }
                const int j = t - C::kLead;
                if (j >= 0 && j < nmax) {
                    const int s = j % kV;
                    const int r = j / kV;
                    if (r > 0 && !mbar_wait(bars + kBarVEmpty + s, (r - 1) & 1, abort_flag)) break;
                    uint8_t *sv = base + C::oV + s * C::kVSlot;
                    uint64_t *bf = bars + kBarVFull + s;
                    mbar_arrive_expect_tx(bf, C::kVBytes);
                    // V^T: keys 64a .. 64a+63 of block j for every channel, two 128-byte-wide boxes
                    tma_load_2d(sv, &tm_v, j * 256, bh * D, bf);
                    tma_load_2d(sv + C::kVAtomBytes, &tm_v, j * 256 + 128, bh * D, bf);
                    v_issued = j + 1;
                }
            }
            drain_wait(bq, 0);
            for (int j = k_issued - kK < 0 ? 0 : k_issued - kK; j < k_issued; ++j)
                drain_wait(bars + kBarKFull + j % kK, (j / kK) & 1);
            for (int j = v_issued - kV < 0 ? 0 : v_issued - kV; j < v_issued; ++j)
                drain_wait(bars + kBarVFull + j % kV, (j / kV) & 1);
        }
    } else {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t kIdQK = idesc_i8(128);
            constexpr uint32_t kIdPV = idesc_f16(D);
            int nqk = 0;
            auto issue_qk = [&](int i, int j) -> bool {
                if (nqk > 0 && !mbar_wait(bars + kBarSEmpty, (nqk - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t qa = base_s + (i ? C::oQ1 : C::oQ0);
                const uint32_t kb = base_s + C::oK + static_cast<uint32_t>(j % kK) * C::kKSlot;
#pragma unroll
                for (int kc = 0; kc < D / 32; ++kc)  // K = 32 int8 per instruction
                    tc_mma_i8(tmem + C::tS, sdesc_kmajor_sw(qa + 32 * kc, C::kQKSbo, C::kQKLayout),
                              sdesc_kmajor_sw(kb + 32 * kc, C::kQKSbo, C::kQKLayout), kIdQK, kc > 0);
                tc_commit(bars + kBarSFull + i);
                ++nqk;
                return true;
            };
            auto issue_pv = [&](int i, int j) -> bool {
                if (!mbar_wait(bars + kBarPFull + i, j & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t pa = base_s + (i ? C::oP1 : C::oP0);
                const uint32_t vb = base_s + C::oV + static_cast<uint32_t>(j % kV) * C::kVSlot;
#pragma unroll
                for (int kc = 0; kc < 8; ++kc) {  // K = 16 halves per instruction, 4 per 64-key atom
                    const uint32_t a = pa + (kc >> 2) * C::kAtomBytes + 32 * (kc & 3);
                    const uint32_t b = vb + (kc >> 2) * C::kVAtomBytes + 32 * (kc & 3);
                    tc_mma_f16(tmem + (i ? C::tO1 : C::tO0), sdesc_kmajor_sw(a, 1024, 2u),
                               sdesc_kmajor_sw(b, 1024, 2u), kIdPV, (j > 0 || kc > 0) ? 1u : 0u);
                }
                tc_commit(bars + kBarPvDone + i);
                return true;
            };

            bool ok = mbar_wait(bars + kBarQ, 0, abort_flag);
            if (ok && nmax > 0) ok = mbar_wait(bars + kBarKFull + 0, 0, abort_flag);
            if (ok && nmax > 0) {
                tc_fence_after();
                if (n0 > 0) ok = issue_qk(0, 0);
                if (ok && n1 > 0) ok = issue_qk(1, 0);
                if (ok) tc_commit(bars + kBarKEmpty + 0);
            }
            for (int j = 0; ok && j < nmax; ++j) {
                if (j + 1 < nmax) {
                    ok = mbar_wait(bars + kBarKFull + (j + 1) % kK, ((j + 1) / kK) & 1, abort_flag);
                    if (!ok) break;
                }
                ok = mbar_wait(bars + kBarVFull + j % kV, (j / kV) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (j + 1 < n0 && !(ok = issue_qk(0, j + 1))) break;
                if (j < n0 && !(ok = issue_pv(0, j))) break;
                if (j + 1 < n1 && !(ok = issue_qk(1, j + 1))) break;
                // K(j + 1) has been read by both S products
                if (j + 1 < nmax) tc_commit(bars + kBarKEmpty + (j + 1) % kK);
                if (j < n1 && !(ok = issue_pv(1, j))) break;
                tc_commit(bars + kBarVEmpty + j % kV);
            }
            tc_commit(bars + kBarDrain);
            drain_wait(bars + kBarDrain, 0);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------------- softmax
        // Warp w: Q tile w/8, column half (w/4)%2, TMEM lanes 32*(w%4)..:
        // one row per thread, two threads per row (as in the FP4 kernel).
        const int i = warp >> 3;
        const int h = (warp >> 2) & 1;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const int tile = i ? tile1 : tile0;
        const int grow = tile * kBlk + r;
        const int n_i = i ? n1 : n0;
        uint64_t *xbar = bars + kBarXch + 4 * i + wq;
        const float c2 = p.scale_log2;
        const float sq = n_i > 0 ? p.q_scale[static_cast<size_t>(bh) * nqt + tile] : 0.0f;
        const float *sk = p.k_scale + static_cast<size_t>(bh) * nkvt;
        const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t tO = (i ? C::tO1 : C::tO0) + h * (D / 2);
        // this half's 64 keys are P atom h: row r at (r/8)*1024 + (r%8)*128
        uint8_t *prow = base + (i ? C::oP1 : C::oP0) + h * C::kAtomBytes + (r >> 3) * 1024 + (r & 7) * 128;
        float *xch = reinterpret_cast<float *>(base + C::oXch);
        float *xl = reinterpret_cast<float *>(base + C::oXl) + (i * 2) * kBlk;
        float m = -INFINITY;
        float l = 0.0f;
        bool ok = true;
        for (int j = 0; j < n_i; ++j) {
            const float skj = sk[j];  // issued before the wait for S, which hides its latency
            if (!warp_wait(bars + kBarSFull + i, j & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t s[2][32];
#pragma unroll
            for (int q = 0; q < 2; ++q) tmem_ld32(trow + C::tS + 64 * h + 32 * q, s[q]);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 2; ++q) reg_fence32(s[q]);
            tc_fence_before();
            mbar_arrive(bars + kBarSEmpty);

            // exact fp32 of the integer scores, in place
#pragma unroll
            for (int e = 0; e < 64; ++e) s[e >> 5][e & 31] = __float_as_uint(i2f_exact(s[e >> 5][e & 31]));
            auto x = [&](int e) -> float { return __uint_as_float(s[e >> 5][e & 31]); };
            const int col0 = j * kBlk + 64 * h;
            const bool tail = col0 + 64 > p.N;
            const bool diag = p.causal && (col0 + 63 > tile * kBlk + off);
            if (tail || diag) {
                int lim = p.N - col0;
                if (p.causal) lim = min(lim, grow + off - col0 + 1);
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (e >= lim) s[e >> 5][e & 31] = __float_as_uint(-INFINITY);
            }
            // partial row maximum: four 3-input chains over 16 scores each
            float mx[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) mx[k] = x(16 * k);
#pragma unroll
            for (int e = 1; e < 15; e += 2) {
#pragma unroll
                for (int k = 0; k < 4; ++k) mx[k] = max3f(mx[k], x(16 * k + e), x(16 * k + e + 1));
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], x(16 * k + 15));
            float *xs = xch + (((j & 1) * 2 + i) * 2) * kBlk;
            xs[h * kBlk + r] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            mbar_arrive(xbar);
            if (!warp_wait(xbar, j & 1, abort_flag)) {
                ok = false;
                break;
            }
            const float rmax = fmaxf(xs[r], xs[kBlk + r]);
            // t = S * f with f = fp32(fp32(s_q s_k) c) > 0 (floored at the
            // smallest normal so that a zero block gives t = +-0, not 0 * inf)
            const float f = fmaxf(__fmul_rn(__fmul_rn(sq, skj), c2), 1.17549435e-38f);
            const float tmax = rmax == -INFINITY ? -INFINITY : __fmul_rn(rmax, f);
            const float m_new = kCross ? fmaxf(fmaxf(m, tmax), -3.402823466e38f) : fmaxf(m, tmax);
            const float nm = -m_new;
            const float alpha = ex2(__fsub_rn(m, m_new));
            // P = 2^(t - m'), fp32 row sum, fp16 P for P V; written to shared
            // memory in two halves of 32 keys (16-byte chunk c of this half,
            // keys 8c .. 8c+7, at chunk c ^ (r % 8)).  The previous P V must
            // have released the buffer first; waiting for it before any P is
            // computed keeps no half in registers across the wait
            const uint64_t ff = pack2(f, f);
            const uint64_t nn = pack2(nm, nm);
            uint64_t acc = pack2(0.0f, 0.0f);
            if (j > 0) {
                if (!warp_wait(bars + kBarPvDone + i, (j - 1) & 1, abort_flag)) ok = false;
                tc_fence_after();
            }
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t ph[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int k = 32 * half + 2 * e;
                    const uint64_t t2 = fma2(pack2(x(k), x(k + 1)), ff, nn);
                    const float p0 = ex2(lo2(t2)), p1 = ex2(hi2(t2));
                    acc = add2(acc, pack2(p0, p1));
                    ph[e] = f16x2(p0, p1);
                }
                if (ok) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int cc = 4 * half + c;
                        *reinterpret_cast<uint4 *>(prow + ((cc ^ (r & 7)) << 4)) =
                            make_uint4(ph[4 * c], ph[4 * c + 1], ph[4 * c + 2], ph[4 * c + 3]);
                    }
                }
            }
            if (!ok) break;
            l = alpha * l + (lo2(acc) + hi2(acc));
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                const uint64_t aa = pack2(alpha, alpha);
#pragma unroll
                for (int q = 0; q < D / 64; ++q) {
                    uint32_t o[32];
                    tmem_ld32(trow + tO + 32 * q, o);
                    tmem_ld_wait();
                    reg_fence32(o);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const uint64_t v = mul2(pack2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), aa);
                        o[e] = __float_as_uint(lo2(v));
                        o[e + 1] = __float_as_uint(hi2(v));
                    }
                    tmem_st32(trow + tO + 32 * q, o);
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bars + kBarPFull + i);
            m = m_new;
        }
        float l_row = 0.0f;
        if (ok && n_i > 0) {
            xl[h * kBlk + r] = l;
            mbar_arrive(xbar);
            ok = warp_wait(xbar, n_i & 1, abort_flag);
            l_row = xl[r] + xl[kBlk + r];
            // log-sum-exp of the row's scaled logits (natural log) for a
            // backward pass: ln 2 (m + log2 l); +inf where no key was seen
            if (ok && p.lse && h == 0 && grow < p.Nq)
                p.lse[static_cast<size_t>(bh) * p.Nq + grow] =
                    l_row > 0.0f ? (m + log2f(l_row)) * 0.693147182f : INFINITY;
        }
        if (ok && n_i > 0 && warp_wait(bars + kBarPvDone + i, (n_i - 1) & 1, abort_flag)) {
            tc_fence_after();
            const float inv = (!kCross || l_row > 0.0f) ? __frcp_rn(l_row) : 0.0f;
            __nv_bfloat16 *orow = p.out + (static_cast<size_t>(bh) * p.Nq + grow) * D + h * (D / 2);
#pragma unroll
            for (int q = 0; q < D / 64; ++q) {
                uint32_t o[32];
                tmem_ld32(trow + tO + 32 * q, o);
                tmem_ld_wait();
                reg_fence32(o);
                if (grow < p.Nq) {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                                        __uint_as_float(o[2 * e + 1]) * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * q);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
        } else if (kCross && ok && n_i == 0 && i <= static_cast<int>(valid1) && grow < p.Nq) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(bh) * p.Nq + grow) * D + h * (D / 2));
#pragma unroll
            for (int v = 0; v < D / 16; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
            if (p.lse && h == 0) p.lse[static_cast<size_t>(bh) * p.Nq + grow] = INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D>
cudaError_t launch_d(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t stream) {
    using C = Cfg<D>;
    auto kernel = p.Nq != p.N ? attn8_fwd_kernel<D, true> : attn8_fwd_kernel<D, false>;
    cudaError_t e = p.Nq != p.N ? smem_attr_once<attn8_fwd_kernel<D, true>>(C::kSmemBytes)
                                : smem_attr_once<attn8_fwd_kernel<D, false>>(C::kSmemBytes);
    if (e != cudaSuccess) return e;
    AttnParams q = p;
    const int nqt = p.Npq / kBlk;
    q.npairs = (nqt + 1) / 2;
    const int total = q.npairs * p.BH;
    const int nsm = sm_count();
    const int rem = total % nsm;
    // (all of them when even that fits in one wave: fewer rows per CTA, lower latency)
    const int split = 2 * total <= nsm ? total : (total > nsm && rem > 0 && 2 * rem <= nsm) ? rem : 0;
    q.pair_units = total - split;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(q.pair_units + 2 * split);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, q);
}

}  // namespace attn8

inline cudaError_t launch_attn_i8(const AttnParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                                  const CUtensorMap &tm_v, int d, cudaStream_t stream) {
    return d == 128 ? attn8::launch_d<128>(p, tm_q, tm_k, tm_v, stream)
                    : attn8::launch_d<64>(p, tm_q, tm_k, tm_v, stream);
}

}  // namespace sa3
