// attn.cuh -- microscaled-FP4 attention forward for sm_100a.
//
// Method ("SageAttention3: Microscaling FP4 Attention ...", abstract; the
// blockwise softmax of "Online normalizer calculation for softmax" and
// FlashAttention, both in its reference list): per 128-row Q block and
// 128-token KV block j,
//   S = Q^ K^_j^T                      block-scaled FP4 MMA, fp32 in TMEM
//   t = S*c, m' = max(m, rowmax t), alpha = 2^(m-m'), P = 2^(t-m')
//   l = alpha*l + rowsum P; P^ = E2M1/E4M3 microscaled P (per 16 columns)
//   O = alpha*O + P^ V^_j              block-scaled FP4 MMA, fp32 in TMEM
// and finally out = bf16(O / l).
//
// One CTA = two 128-row Q tiles of one (b, h), 18 warps:
//   warps 0-7  softmax for Q tile 0: warp w owns TMEM lanes 32*(w%4) ..
//              (one row per thread) and column half (w/4)%2, so each row
//              is shared by two threads that exchange partial row maxima
//   warps 8-15 softmax for Q tile 1
//   warp 16    producer: TMA loads of Q, and of K / V^T codes + scales into
//              a 6-stage ring (mbarrier transaction counts).  A slot stays
//              held from S = Q K^T until O += P V of both tiles, about two
//              blocks, so the ring runs four blocks ahead of the MMAs; at
//              d = 128 six stages were 1.5-2 % faster than three, and seven
//              or eight no faster (the Q-on-load instance has room for six)
//   warp 17    allocates TMEM and issues every tcgen05 op from one thread:
//              scale-factor copies (tcgen05.cp), S = Q K^T, O += P V
// TMEM (512 columns): S (128, shared by both tiles -- each softmax group
// loads it to registers at once and releases it), O0, O1 (d each), and
// the scale factors of Q0, Q1, K, P and V.  tcgen05.cp and tcgen05.mma
// from one thread execute in issue order, so each scale-factor region is
// rewritten right before the MMA that reads it.  P goes through shared
// memory (64-byte swizzled K-major rows + 512-byte scale atoms) because
// the block-scaled FP4 MMA takes A from shared memory only.
// The tensor pipe order per KV block j is QK0(j+1), PV0(j), QK1(j+1),
// PV1(j): each softmax group finds its next S ready as soon as it has
// produced its P, so the two groups run concurrently and the exp / FMA
// pipes (the bottleneck on B200) stay busy.
#pragma once

#include "quant.cuh"
#include "sa3_internal.h"
#include "sm100.cuh"

namespace sa3 {
namespace attn {

constexpr int kBlk = 128;
constexpr int kStages = 6;
constexpr int kSoftmaxWarps = 16;               // 2 tiles x 2 column halves x 4 lane quadrants
constexpr int kWarpProducer = kSoftmaxWarps;     // warp 16
constexpr int kWarpMma = kSoftmaxWarps + 1;      // warp 17
// 576 threads.  Warps are placed on the SM's four sub-partitions in turn, so
// two of them hold 5 warps; a sub-partition's 16384 registers then allow 96
// per thread (allocation granularity 8), which is what the launch bound
// gives the compiler, and what the kernel uses
constexpr int kThreads = (kSoftmaxWarps + 2) * 32;

constexpr int kBarCountBytes = (18 + 2 * kStages) * 8;  // barrier slots below

template <int D>
struct Cfg {
    static constexpr int al(int x) { return (x + 1023) & ~1023; }
    static constexpr int kRowB = D / 2;                 // bytes per Q/K code row
    static constexpr int kQBytes = kBlk * kRowB;
    static constexpr int kSfBytes = (D / 64) * 512;    // Q or K tile scales
    static constexpr int kVBytes = D * 64;             // V^T tile: D rows x 128 tokens
    static constexpr int kVsfBytes = 1024;
    static constexpr int kPBytes = kBlk * 64;
    static constexpr int kPsfBytes = 1024;
    static constexpr uint32_t kQKLayout = (D == 128) ? 4u : 6u;  // 64B / 32B swizzle
    static constexpr uint32_t kQKSbo = 8 * kRowB;
    // shared memory map, offsets from a 1024-byte aligned base
    static constexpr int oQ0 = 0;
    static constexpr int oQ1 = al(oQ0 + kQBytes);
    static constexpr int oQsf0 = al(oQ1 + kQBytes);
    static constexpr int oQsf1 = oQsf0 + kSfBytes;
    static constexpr int oStage = al(oQsf1 + kSfBytes);
    static constexpr int sK = 0;
    static constexpr int sV = al(kQBytes);
    static constexpr int sKsf = sV + al(kVBytes);
    static constexpr int sVsf = sKsf + kSfBytes;
    static constexpr int kStageBytes = al(sVsf + kVsfBytes);
    static constexpr int oP0 = oStage + kStages * kStageBytes;
    static constexpr int oP1 = oP0 + kPBytes;
    static constexpr int oPsf0 = oP1 + kPBytes;
    static constexpr int oPsf1 = oPsf0 + kPsfBytes;
    static constexpr int oLut = oPsf1 + kPsfBytes;     // 2 x 256 floats: log2(2^pre / s), s per E4M3 code s
    static constexpr int oXch = oLut + 2048;           // row maxima [2 parity][2 tiles][2 halves][128]
    static constexpr int oXl = oXch + 4096;            // row sums [2 tiles][2 halves][128]
    static constexpr int oBar = oXl + 2048;
    static constexpr int kSmemBytes = oBar + 256 + 1024;
    // Q quantized on load (kQLoad instances only): bf16 staging of the two Q
    // tiles (D/64 boxes of 64 channels x 128 tokens each, 128-byte swizzle,
    // as the quantizer stages them) and 1/s per E4M3 scale code
    static constexpr int kQbfBytes = kBlk * D * 2;
    static constexpr int oQbf = al(oBar + 256);
    static constexpr int oRcp = oQbf + 2 * kQbfBytes;
    static constexpr int kSmemBytesQL = oRcp + 1024 + 1024;
    static_assert(kSmemBytesQL <= 227 * 1024, "shared memory budget (Q on load)");
    // TMEM columns
    static constexpr uint32_t tS = 0;
    static constexpr uint32_t tO0 = 128;
    static constexpr uint32_t tO1 = 128 + D;
    static constexpr uint32_t tSfq0 = 128 + 2 * D;
    static constexpr uint32_t tSfq1 = tSfq0 + 4 * (D / 64);
    static constexpr uint32_t tSfk = tSfq1 + 4 * (D / 64);
    static constexpr uint32_t tSfp = tSfk + 4 * (D / 64);
    static constexpr uint32_t tSfv = tSfp + 8;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(tSfv + 8 <= kTmemCols, "TMEM budget");
    static_assert(kBarCountBytes + 8 <= 256, "barrier area");
};

// Barrier slots (uint64 each) after oBar.
enum : int {
    kBarQ = 0,
    kBarKvFull = 1,                  // kStages
    kBarKvEmpty = 1 + kStages,       // kStages
    kBarSFull = 1 + 2 * kStages,     // 2
    kBarSEmpty = 3 + 2 * kStages,    // 1
    kBarPFull = 4 + 2 * kStages,     // 2
    kBarPvDone = 6 + 2 * kStages,    // 2
    kBarDrain = 8 + 2 * kStages,     // 1
    kBarXch = 9 + 2 * kStages,       // 8: [tile][lane quadrant], 64 arrivals
    kBarQReady = 17 + 2 * kStages,   // 1 (Q on load): the 512 softmax threads have quantized Q
    kBarCount = 18 + 2 * kStages
};
static_assert(kBarCount * 8 == kBarCountBytes, "barrier slots");

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kSixth = 1.0f / 6.0f;

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// E4M3 codes of two floats: byte 0 from `lo`, byte 1 from `hi`.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(hi), "f"(lo));
    return out;
}

// mbar_wait with a warp-uniform result, for code that continues with
// .sync.aligned tcgen05 instructions.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain copies in
// flight before the CTA exits).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kWaitLimitNs) {
            atomicOr(&g_sa3_status, 1u);
            return;
        }
    }
}

// Quantizes one staged bf16 Q tile in shared memory (this thread: token
// row qk_row(t), channel half qk_part(t) of the tile's 256 threads) into
// the layout the MMA reads: E2M1 codes in 64-byte (D = 128) or 32-byte
// (D = 64) swizzled K-major rows, scales in 512-byte atoms.  The blocks are quantized by the
// quantizer's own routine; rows past Nq arrive as zeros and get code 0,
// scale 0.
template <int D>
__device__ __forceinline__ void quantize_q_tile(const uint8_t *__restrict__ stage, const float *__restrict__ rcp_lut,
                                                uint8_t *__restrict__ codes, uint8_t *__restrict__ sf, int t) {
    const int row = quant::qk_row(t);
    const int part = quant::qk_part(t);
    uint32_t cw[D / 16];
    const uint32_t scw = quant::row_part_codes<D>(stage, row, part, false, nullptr, rcp_lut, cw);
    if constexpr (D == 128) {
        // 64-byte rows; 16-byte chunks 2*part, 2*part+1, chunk index XOR (row/2)%4
        uint8_t *prow = codes + row * 64;
        const int sw = (row >> 1) & 3;
        *reinterpret_cast<uint4 *>(prow + (((2 * part) ^ sw) << 4)) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4 *>(prow + (((2 * part + 1) ^ sw) << 4)) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
        *reinterpret_cast<uint32_t *>(sf + part * 512 + quant::atom_off(row, 0)) = scw;
    } else {
        // 32-byte rows; 16-byte chunk `part`, chunk index XOR (row/4)%2
        *reinterpret_cast<uint4 *>(codes + row * 32 + ((part ^ ((row >> 2) & 1)) << 4)) =
            make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint16_t *>(sf + quant::atom_off(row, 2 * part)) = static_cast<uint16_t>(scw);
    }
}

// kCross: query and key/value lengths differ (bottom-right causal offset,
// rows that may see no key).  kTwo: P is pre-scaled by 2^11 before it is
// microscaled (two-level P).  kQLoad: Q arrives as bf16 and the softmax
// warps quantize it before the first S (tm_q is then the 3-D bf16 map).
// Each term is compiled only into the instances that use it.
template <int D, bool kCross, bool kTwo, bool kQLoad>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_s - raw_s);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + C::oBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kBarCount);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Work unit -> (b*H+h, Q tiles).  Units [0, pair_units) are pairs of
    // Q tiles, ordered by rank (heaviest pairs first when causal) and then
    // head; the pairs after them are split into single-tile units that fill
    // what would otherwise be a short last wave.
    const int nqt = p.Npq / kBlk;   // Q tiles
    const int nkvt = p.Np / kBlk;   // KV blocks
    const int off = kCross ? p.N - p.Nq : 0;  // causal: row r sees keys 0 .. r + off
    const int u = static_cast<int>(blockIdx.x);
    const bool single = u >= p.pair_units;
    const int pu = single ? p.pair_units + (u - p.pair_units) / 2 : u;
    const int bh = pu % p.BH;
    const int rank = pu / p.BH;
    const int pair = p.causal ? p.npairs - 1 - rank : rank;
    const int tile0 = 2 * pair + (single ? ((u - p.pair_units) & 1) : 0);
    const int tile1 = tile0 + 1;
    if (tile0 >= nqt) return;  // second half of a split pair whose head has an odd tile count
    const bool valid1 = !single && tile1 < nqt;
    // KV blocks up to the last key any row of the tile sees (0: none)
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
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bars + kBarKvFull + s, 1);
            mbar_init(bars + kBarKvEmpty + s, 1);
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
        mbar_init(bars + kBarQReady, 16 * 32);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < 256) {
        // per E4M3 scale code: log2(1/s) and s.  Code 0 (and the NaN codes,
        // which the saturating conversion never produces) map to log2 = 0,
        // s = 1: such a block holds only P < 6 * 2^-10, whose codes at scale
        // 1 are all 0, exactly as at scale 0, and whose row-sum terms stay P.
        // kTwo: every log2 entry gains the pre-scale exponent 11, so that
        // y = P * 2^11 / s (and y = P * 2^11 for code 0, whose P' is still
        // below 6 * 2^-10 and quantizes to 0)
        const float v = e4m3_value(threadIdx.x);
        const bool unit = v == 0.0f || v != v;
        const float pre = kTwo ? 11.0f : 0.0f;
        reinterpret_cast<float *>(base + C::oLut)[threadIdx.x] = unit ? pre : pre - log2f(v);
        reinterpret_cast<float *>(base + C::oLut)[256 + threadIdx.x] = unit ? 1.0f : v;
        if constexpr (kQLoad)
            reinterpret_cast<float *>(base + C::oRcp)[threadIdx.x] = unit ? 0.0f : __frcp_rn(v);  // 1/s, exact
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
    const float *lg_lut = reinterpret_cast<const float *>(base + C::oLut);
    const float *sv_lut = lg_lut + 256;

    if (warp >= kWarpProducer) {
      if (warp == kWarpProducer) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            uint64_t *bq = bars + kBarQ;
            if constexpr (kQLoad) {
                // bf16 Q tiles, boxes of 64 channels x 128 tokens (tokens past Nq read as 0)
                const uint64_t pol = l2_policy_evict_first();
                mbar_arrive_expect_tx(bq, (valid1 ? 2u : 1u) * C::kQbfBytes);
                for (int i = 0; i <= static_cast<int>(valid1); ++i)
#pragma unroll
                    for (int b = 0; b < D / 64; ++b)
                        tma_load_3d_hint(base + C::oQbf + i * C::kQbfBytes + b * (kBlk * 128), &tm_q, b * 64,
                                         (i ? tile1 : tile0) * kBlk, bh, bq, pol);
            } else {
                mbar_arrive_expect_tx(bq, (valid1 ? 2u : 1u) * (C::kQBytes + C::kSfBytes));
                tma_load_2d(base + C::oQ0, &tm_q, 0, bh * p.Npq + tile0 * kBlk, bq);
                bulk_load(base + C::oQsf0, p.q_sf + static_cast<size_t>(bh * nqt + tile0) * C::kSfBytes, C::kSfBytes,
                          bq);
                if (valid1) {
                    tma_load_2d(base + C::oQ1, &tm_q, 0, bh * p.Npq + tile1 * kBlk, bq);
                    bulk_load(base + C::oQsf1, p.q_sf + static_cast<size_t>(bh * nqt + tile1) * C::kSfBytes,
                              C::kSfBytes, bq);
                }
            }
            int issued = 0;
            for (int j = 0; j < nmax; ++j) {
                const int s = j % kStages;
                const int u = j / kStages;
                if (u > 0 && !mbar_wait(bars + kBarKvEmpty + s, (u - 1) & 1, abort_flag)) break;
                uint8_t *st = base + C::oStage + s * C::kStageBytes;
                uint64_t *bf = bars + kBarKvFull + s;
                mbar_arrive_expect_tx(bf, C::kQBytes + C::kSfBytes + C::kVBytes + C::kVsfBytes);
                tma_load_2d(st + C::sK, &tm_k, 0, bh * p.Np + j * kBlk, bf);
                bulk_load(st + C::sKsf, p.k_sf + static_cast<size_t>(bh * nkvt + j) * C::kSfBytes, C::kSfBytes, bf);
                tma_load_2d(st + C::sV, &tm_v, j * 64, bh * D, bf);
                bulk_load(st + C::sVsf, p.vt_sf + (static_cast<size_t>(bh) * (p.Np / 64) + 2 * j) * 512, C::kVsfBytes,
                          bf);
                issued = j + 1;
            }
            // Let every copy this thread started land before the CTA exits.
            drain_wait(bq, 0);
            for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j)
                drain_wait(bars + kBarKvFull + j % kStages, (j / kStages) & 1);
        }
    } else {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            // This thread shares its SM sub-partition with four busy softmax
            // warps, so its instruction stream is kept short: shared-memory
            // descriptors are built from precomputed low words (address >> 4
            // | leading offset << 16) and a per-operand-kind high word, and
            // ring positions advance incrementally.
            constexpr uint32_t idesc_qk = idesc_mxf4nvf4(128, 128);
            constexpr uint32_t idesc_pv = idesc_mxf4nvf4(128, D);
            constexpr uint32_t kHiQK = (static_cast<uint32_t>(C::kQKSbo) >> 4) | (1u << 14) | (C::kQKLayout << 29);
            constexpr uint32_t kHiPV = (512u >> 4) | (1u << 14) | (4u << 29);
            constexpr uint32_t kHiSF = (128u >> 4) | (1u << 14);
            constexpr uint32_t kStageLo = static_cast<uint32_t>(C::kStageBytes) >> 4;
            auto lo_of = [](uint32_t saddr, uint32_t lead) -> uint32_t {
                return ((saddr >> 4) & 0x3FFFu) | (lead << 16);
            };
            auto desc = [](uint32_t lo, uint32_t hi) -> uint64_t {
                uint64_t d;
                asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
                return d;
            };
            const uint32_t st0 = base_s + C::oStage;
            const uint32_t k_lo0 = lo_of(st0 + C::sK, 1), v_lo0 = lo_of(st0 + C::sV, 1);
            const uint32_t ksf_lo0 = lo_of(st0 + C::sKsf, 8), vsf_lo0 = lo_of(st0 + C::sVsf, 8);
            const uint32_t q_lo0 = lo_of(base_s + C::oQ0, 1), q_lo1 = lo_of(base_s + C::oQ1, 1);
            const uint32_t p_lo0 = lo_of(base_s + C::oP0, 1), p_lo1 = lo_of(base_s + C::oP1, 1);
            const uint32_t psf_lo0 = lo_of(base_s + C::oPsf0, 8), psf_lo1 = lo_of(base_s + C::oPsf1, 8);
            const uint32_t t_s = tmem + C::tS, t_sfk = tmem + C::tSfk, t_sfp = tmem + C::tSfp, t_sfv = tmem + C::tSfv;
            int nqk = 0;
            auto copy_ksf = [&](int s) {
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tc_cp_32x128b_warpx4(t_sfk + 4 * a, desc(ksf_lo0 + s * kStageLo + 32 * a, kHiSF));
            };
            auto issue_qk = [&](int i, int s) -> bool {
                if (nqk > 0 && !mbar_wait(bars + kBarSEmpty, (nqk - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t qa = i ? q_lo1 : q_lo0;
                const uint32_t kb = k_lo0 + s * kStageLo;
                const uint32_t sfq = tmem + (i ? C::tSfq1 : C::tSfq0);
#pragma unroll
                for (int kc = 0; kc < D / 64; ++kc)
                    tc_mma_mxf4nvf4(t_s, desc(qa + 2 * kc, kHiQK), desc(kb + 2 * kc, kHiQK), idesc_qk, sfq + 4 * kc,
                                    t_sfk + 4 * kc, kc > 0);
                tc_commit(bars + kBarSFull + i);
                ++nqk;
                return true;
            };
            auto issue_pv = [&](int i, int j, int s, bool load_vsf) -> bool {
                if (!mbar_wait(bars + kBarPFull + i, j & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t pa = i ? p_lo1 : p_lo0;
                const uint32_t psf = i ? psf_lo1 : psf_lo0;
                const uint32_t vb = v_lo0 + s * kStageLo;
                tc_cp_32x128b_warpx4(t_sfp, desc(psf, kHiSF));
                tc_cp_32x128b_warpx4(t_sfp + 4, desc(psf + 32, kHiSF));
                if (load_vsf) {
                    const uint32_t vsf = vsf_lo0 + s * kStageLo;
                    tc_cp_32x128b_warpx4(t_sfv, desc(vsf, kHiSF));
                    tc_cp_32x128b_warpx4(t_sfv + 4, desc(vsf + 32, kHiSF));
                }
                const uint32_t t_o = tmem + (i ? C::tO1 : C::tO0);
#pragma unroll
                for (int kc = 0; kc < 2; ++kc)
                    tc_mma_mxf4nvf4(t_o, desc(pa + 2 * kc, kHiPV), desc(vb + 2 * kc, kHiPV), idesc_pv, t_sfp + 4 * kc,
                                    t_sfv + 4 * kc, (j > 0 || kc > 0) ? 1u : 0u);
                tc_commit(bars + kBarPvDone + i);
                return true;
            };

            bool ok = mbar_wait(bars + (kQLoad ? kBarQReady : kBarQ), 0, abort_flag);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int a = 0; a < D / 64; ++a) {
                    tc_cp_32x128b_warpx4(tmem + C::tSfq0 + 4 * a, sdesc_sf_atom(base_s + C::oQsf0 + 512 * a));
                    if (valid1)
                        tc_cp_32x128b_warpx4(tmem + C::tSfq1 + 4 * a, sdesc_sf_atom(base_s + C::oQsf1 + 512 * a));
                }
                if (nmax > 0) ok = mbar_wait(bars + kBarKvFull + 0, 0, abort_flag);
            }
            if (ok && nmax > 0) {
                tc_fence_after();
                copy_ksf(0);
                if (n0 > 0) ok = issue_qk(0, 0);
                if (ok && n1 > 0) ok = issue_qk(1, 0);
            }
            // s: ring stage of block j; s1, ph1: stage and parity of block j + 1
            int s = 0, s1 = kStages > 1 ? 1 : 0;
            uint32_t ph1 = kStages > 1 ? 0u : 1u;
            for (int j = 0; ok && j < nmax; ++j) {
                if (j + 1 < nmax) {
                    ok = mbar_wait(bars + kBarKvFull + s1, ph1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    copy_ksf(s1);
                }
                if (j + 1 < n0 && !(ok = issue_qk(0, s1))) break;
                if (j < n0 && !(ok = issue_pv(0, j, s, true))) break;
                if (j + 1 < n1 && !(ok = issue_qk(1, s1))) break;
                if (j < n1 && !(ok = issue_pv(1, j, s, !(j < n0)))) break;
                tc_commit(bars + kBarKvEmpty + s);
                s = s1;
                if (++s1 == kStages) {
                    s1 = 0;
                    ph1 ^= 1u;
                }
            }
            // Every tcgen05 op issued above completes before TMEM is freed.
            tc_commit(bars + kBarDrain);
            drain_wait(bars + kBarDrain, 0);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------------- softmax
        // Warp w: Q tile w/8, column half (w/4)%2 (64 of the 128 S columns,
        // D/2 of the O columns), TMEM lanes 32*(w%4) .. : one row per thread,
        // two threads per row.  The two halves of a row exchange their
        // partial row maxima through shared memory (double-buffered by KV
        // block parity), ordered by an mbarrier of 64 arrivals per pair of
        // warps (bounded waits); each half keeps the row sum of its columns,
        // added once at the end through the same barrier.
        const int i = warp >> 3;         // Q tile of this warp
        const int h = (warp >> 2) & 1;   // column half
        const int wq = warp & 3;         // TMEM lane quadrant = rows 32*wq ..
        const int r = wq * 32 + lane;    // row inside the tile
        const int tile = i ? tile1 : tile0;
        const int grow = tile * kBlk + r;
        const int n_i = i ? n1 : n0;
        uint64_t *xbar = bars + kBarXch + 4 * i + wq;  // the two warps sharing these rows
        const float c2 = p.scale_log2;
        const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t tO = (i ? C::tO1 : C::tO0) + h * (D / 2);
        uint8_t *P = base + (i ? C::oP1 : C::oP0);
        uint8_t *Psf = base + (i ? C::oPsf1 : C::oPsf0);
        float *xch = reinterpret_cast<float *>(base + C::oXch);  // [parity][tile][half][row]
        float *xl = reinterpret_cast<float *>(base + C::oXl) + (i * 2) * kBlk;  // [tile][half][row]
        float m = -INFINITY;
        float l = 0.0f;
        bool ok = true;
        if constexpr (kQLoad) {
            // Q on load: the 256 threads of tile i quantize its staged bf16
            // tile into the Q code and scale buffers the MMA reads
            ok = warp_wait(bars + kBarQ, 0, abort_flag);
            if (ok && (i == 0 || valid1))
                quantize_q_tile<D>(base + C::oQbf + i * C::kQbfBytes, reinterpret_cast<const float *>(base + C::oRcp),
                                   base + (i ? C::oQ1 : C::oQ0), base + (i ? C::oQsf1 : C::oQsf0),
                                   static_cast<int>(threadIdx.x) & 255);
            fence_proxy_async_smem();
            mbar_arrive(bars + kBarQReady);
        }
        for (int j = 0; ok && j < n_i; ++j) {
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

            const int col0 = j * kBlk + 64 * h;
            const bool tail = col0 + 64 > p.N;
            const bool diag = p.causal && (col0 + 63 > tile * kBlk + off);
            if (tail || diag) {
                // columns col0 + k with k >= lim are masked for this row
                int lim = p.N - col0;
                if (p.causal) lim = min(lim, grow + off - col0 + 1);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * q + e >= lim) s[q][e] = __float_as_uint(-INFINITY);
                }
            }
            // block maxima of the raw scores (c > 0, so max commutes with * c)
            float bm[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t *x = &s[b >> 1][(b & 1) * 16];
                const float m0 = max3f(__uint_as_float(x[0]), __uint_as_float(x[1]), __uint_as_float(x[2]));
                const float m1 = max3f(__uint_as_float(x[3]), __uint_as_float(x[4]), __uint_as_float(x[5]));
                const float m2 = max3f(__uint_as_float(x[6]), __uint_as_float(x[7]), __uint_as_float(x[8]));
                const float m3 = max3f(__uint_as_float(x[9]), __uint_as_float(x[10]), __uint_as_float(x[11]));
                const float m4 = max3f(__uint_as_float(x[12]), __uint_as_float(x[13]), __uint_as_float(x[14]));
                bm[b] = max3f(max3f(m0, m1, m2), max3f(m3, m4, __uint_as_float(x[15])), m0);
            }
            float *xs = xch + (((j & 1) * 2 + i) * 2) * kBlk;
            xs[h * kBlk + r] = max3f(bm[0], bm[1], fmaxf(bm[2], bm[3]));
            mbar_arrive(xbar);
            if (!warp_wait(xbar, j & 1, abort_flag)) {
                ok = false;
                break;
            }
            const float rmax = fmaxf(xs[r], xs[kBlk + r]);
            // (kCross) clamped below at -FLT_MAX: a row that has seen no key yet
            // gets P = 0 and alpha = 0 (its O and l are still 0), never inf - inf
            const float m_new = kCross ? fmaxf(fmaxf(m, __fmul_rn(rmax, c2)), -3.402823466e38f)
                                       : fmaxf(m, __fmul_rn(rmax, c2));
            // -m' plus the optional two-level pre-scale exponent (0 or 11):
            // P' = P * 2^pre is what gets microscaled; l and O both carry the
            // 2^pre, so O / l needs no correction
            const float nm = -m_new;
            const float alpha = ex2(__fsub_rn(m, m_new));
            // block scales: s_b = E4M3(amax_b / 6) with amax_b = 2^(bm_b*c - m'),
            // two blocks per conversion
            uint32_t scw;
            float lg[4], sv[4];
#pragma unroll
            for (int b = 0; b < 4; b += 2) {
                const float a0 = ex2(__fadd_rn(__fmul_rn(bm[b], c2), nm));
                const float a1 = ex2(__fadd_rn(__fmul_rn(bm[b + 1], c2), nm));
                // amax' / 6 with amax' = 2^11 * amax under kTwo (exact: 2^11 * fp32(1/6))
                constexpr float kDiv = kTwo ? 2048.0f * kSixth : kSixth;
                const uint32_t sc2 = cvt_e4m3x2(a1 * kDiv, a0 * kDiv);  // byte 0: block b
                lg[b] = lg_lut[sc2 & 0xFF];
                lg[b + 1] = lg_lut[sc2 >> 8];
                sv[b] = sv_lut[sc2 & 0xFF];
                sv[b + 1] = sv_lut[sc2 >> 8];
                if (b == 0) scw = sc2;
                else scw |= sc2 << 16;
            }
            // y = P / s_b = 2^(t - m' + log2(1/s_b)) (the 1/s_b folded into the
            // exponent), codes of y; the row sum of P is sum_b s_b * sum(y)
            const uint64_t cc = pack2(c2, c2);
            float sum = 0.0f;
            uint32_t pc[8];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t *x = &s[b >> 1][(b & 1) * 16];
                const float bias = __fadd_rn(nm, lg[b]);
                const uint64_t bb = pack2(bias, bias);
                uint64_t vy[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint64_t t2 = fma2(pack2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), cc, bb);
                    vy[e] = pack2(ex2(lo2(t2)), ex2(hi2(t2)));
                }
                const uint64_t s01 = add2(add2(vy[0], vy[1]), add2(vy[2], vy[3]));
                const uint64_t s23 = add2(add2(vy[4], vy[5]), add2(vy[6], vy[7]));
                const uint64_t sb = add2(s01, s23);
                sum = fmaf(sv[b], lo2(sb) + hi2(sb), sum);
                pc[2 * b] = cvt_e2m1x8(lo2(vy[0]), hi2(vy[0]), lo2(vy[1]), hi2(vy[1]), lo2(vy[2]), hi2(vy[2]),
                                       lo2(vy[3]), hi2(vy[3]));
                pc[2 * b + 1] = cvt_e2m1x8(lo2(vy[4]), hi2(vy[4]), lo2(vy[5]), hi2(vy[5]), lo2(vy[6]), hi2(vy[6]),
                                           lo2(vy[7]), hi2(vy[7]));
            }
            l = alpha * l + sum;

            // P buffer and O are free once the previous P V has completed.
            if (j > 0) {
                if (!warp_wait(bars + kBarPvDone + i, (j - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            {
                // this half's 32 code bytes = 16-byte chunks 2h, 2h+1 of the 64-byte row
                uint8_t *prow = P + (r >> 3) * 512 + (r & 7) * 64;
                const int sw = (r & 7) >> 1;
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    *reinterpret_cast<uint4 *>(prow + (((2 * h + c) ^ sw) << 4)) =
                        make_uint4(pc[4 * c], pc[4 * c + 1], pc[4 * c + 2], pc[4 * c + 3]);
                // blocks 4h .. 4h+3 = the four columns of scale atom h
                *reinterpret_cast<uint32_t *>(Psf + 512 * h + 16 * (r & 31) + 4 * (r >> 5)) = scw;
            }
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
                // O = alpha * O for this warp's 32 rows, this half's D/2 columns
                uint32_t o[D / 64][32];
#pragma unroll
                for (int q = 0; q < D / 64; ++q) tmem_ld32(trow + tO + 32 * q, o[q]);
                tmem_ld_wait();
                const uint64_t aa = pack2(alpha, alpha);
#pragma unroll
                for (int q = 0; q < D / 64; ++q) {
                    reg_fence32(o[q]);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const uint64_t v = mul2(pack2(__uint_as_float(o[q][e]), __uint_as_float(o[q][e + 1])), aa);
                        o[q][e] = __float_as_uint(lo2(v));
                        o[q][e + 1] = __float_as_uint(hi2(v));
                    }
                    tmem_st32(trow + tO + 32 * q, o[q]);
                }
                tmem_st_wait();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bars + kBarPFull + i);
            m = m_new;
        }
        // row sum = the sums of the two halves, exchanged through the pair's
        // barrier once more (phase n_i)
        float l_row = 0.0f;
        if (ok && n_i > 0) {
            xl[h * kBlk + r] = l;
            mbar_arrive(xbar);
            ok = warp_wait(xbar, n_i & 1, abort_flag);
            l_row = xl[r] + xl[kBlk + r];
        }
        if (ok && n_i > 0 && warp_wait(bars + kBarPvDone + i, (n_i - 1) & 1, abort_flag)) {
            tc_fence_after();
            // a row that sees no key (kCross only) outputs 0
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
                    if (p.v_mean) {
                        // V smoothing: the mean of V comes back after O / l (a
                        // row that sees no key stays 0)
                        const float4 *vm = reinterpret_cast<const float4 *>(
                            p.v_mean + static_cast<size_t>(bh) * D + h * (D / 2) + 32 * q);
                        const bool live = !kCross || l_row > 0.0f;
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 m4 = live ? vm[e4] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                            const __nv_bfloat162 a = __floats2bfloat162_rn(
                                __fadd_rn(__uint_as_float(o[4 * e4]) * inv, m4.x),
                                __fadd_rn(__uint_as_float(o[4 * e4 + 1]) * inv, m4.y));
                            const __nv_bfloat162 b = __floats2bfloat162_rn(
                                __fadd_rn(__uint_as_float(o[4 * e4 + 2]) * inv, m4.z),
                                __fadd_rn(__uint_as_float(o[4 * e4 + 3]) * inv, m4.w));
                            w[2 * e4] = *reinterpret_cast<const uint32_t *>(&a);
                            w[2 * e4 + 1] = *reinterpret_cast<const uint32_t *>(&b);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                                            __uint_as_float(o[2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * q);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
        } else if (kCross && ok && n_i == 0 && i <= static_cast<int>(valid1) && grow < p.Nq) {
            // causal with more queries than keys: no row of this tile sees a key
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(bh) * p.Nq + grow) * D + h * (D / 2));
#pragma unroll
            for (int v = 0; v < D / 16; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int D, bool kQLoad>
cudaError_t launch_dq(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                      cudaStream_t stream) {
    using C = Cfg<D>;
    constexpr int smem = kQLoad ? C::kSmemBytesQL : C::kSmemBytes;
    const bool cross = p.Nq != p.N;
    const bool two = p.p_pre_log2 != 0.0f;
    auto kernel = cross ? (two ? attn_fwd_kernel<D, true, true, kQLoad> : attn_fwd_kernel<D, true, false, kQLoad>)
                        : (two ? attn_fwd_kernel<D, false, true, kQLoad> : attn_fwd_kernel<D, false, false, kQLoad>);
    cudaError_t e = cross ? (two ? smem_attr_once<attn_fwd_kernel<D, true, true, kQLoad>>(smem)
                                 : smem_attr_once<attn_fwd_kernel<D, true, false, kQLoad>>(smem))
                          : (two ? smem_attr_once<attn_fwd_kernel<D, false, true, kQLoad>>(smem)
                                 : smem_attr_once<attn_fwd_kernel<D, false, false, kQLoad>>(smem));
    if (e != cudaSuccess) return e;
    // Split the pairs of a last wave that would fill at most half of the SMs
    // into single-tile units (one CTA per SM).
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
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, q);
}

template <int D>
cudaError_t launch_d(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t stream) {
    return p.q_load ? launch_dq<D, true>(p, tq, tk, tv, stream) : launch_dq<D, false>(p, tq, tk, tv, stream);
}

}  // namespace attn

inline cudaError_t launch_attn(const AttnParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                               const CUtensorMap &tm_v, int d, cudaStream_t stream) {
    return d == 128 ? attn::launch_d<128>(p, tm_q, tm_k, tm_v, stream)
                    : attn::launch_d<64>(p, tm_q, tm_k, tm_v, stream);
}

}  // namespace sa3
