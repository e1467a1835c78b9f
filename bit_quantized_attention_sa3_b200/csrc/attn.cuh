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
// Persistent kernel: one CTA per SM walks a static list of 128-row Q tiles
// (work units); the KV blocks of all its tiles form one sequence g = 0, 1,
// 2, ...  14 warps:
//   warps 0-3   softmax warpgroup A: the blocks with even g
//   warps 4-7   softmax warpgroup B: the blocks with odd g
//               (one thread per row: warp w owns TMEM lanes 32*(w%4) ..)
//   warps 8-11  correction warpgroup: rescales O by alpha between two P V
//               products and writes the tile's output (O / l -> bf16)
//   warp 12     producer: TMA loads of Q (two tile slots) and of K / V^T
//               codes + scales (a ring of stages)
//   warp 13     allocates TMEM and issues every tcgen05 op from one thread
// TMEM: S_A, S_B (128 columns each: block g lands in S_(g%2)), O (d), and
// the scale factors of Q (two tile slots), K, P and V.  Because the two
// warpgroups work on different blocks, one can take exponentials while the
// other loads its S, forms its row maxima or waits for the next S, which
// keeps the exp2 unit (the bound of this kernel) busy.  The running maximum
// passes from block g-1 to block g through shared memory; alpha goes to the
// correction warps through a ring of four slots.  tcgen05.cp and
// tcgen05.mma issued by one thread execute in order, so each scale-factor
// region is rewritten right before the MMA that reads it.  P goes through
// shared memory (64-byte swizzled K-major rows + 512-byte scale atoms)
// because the block-scaled FP4 MMA takes A from shared memory only.
#pragma once

#include "sa3_internal.h"
#include "sm100.cuh"

namespace sa3 {
namespace attn {

constexpr int kBlk = 128;
constexpr int kWarpCorr = 8;       // warps 8-11
constexpr int kWarpProducer = 12;
constexpr int kWarpMma = 13;
constexpr int kThreads = 14 * 32;  // 448 threads: at most 144 registers each

template <int D>
struct Cfg {
    static constexpr int al(int x) { return (x + 1023) & ~1023; }
    static constexpr int kStages = D == 128 ? 6 : 8;   // K/V ring
    static constexpr int kRowB = D / 2;                 // bytes per Q/K code row
    static constexpr int kQBytes = kBlk * kRowB;
    static constexpr int kSfBytes = (D / 64) * 512;    // Q or K tile scales
    static constexpr int kVBytes = D * 64;             // V^T tile: D rows x 128 tokens
    static constexpr int kVsfBytes = 1024;
    static constexpr int kPBytes = kBlk * 64;
    static constexpr int kPsfBytes = 1024;
    static constexpr int kQSlot = (kQBytes + 1023) & ~1023;  // one Q tile slot
    static constexpr uint32_t kQKLayout = (D == 128) ? 4u : 6u;  // 64B / 32B swizzle
    static constexpr uint32_t kQKSbo = 8 * kRowB;
    // shared memory map, offsets from a 1024-byte aligned base
    static constexpr int oQ = 0;                                 // 2 tile slots
    static constexpr int oQsf = oQ + 2 * kQSlot;                 // 2 x kSfBytes
    static constexpr int oStage = al(oQsf + 2 * kSfBytes);
    static constexpr int sK = 0;
    static constexpr int sV = al(kQBytes);
    static constexpr int sKsf = sV + al(kVBytes);
    static constexpr int sVsf = sKsf + kSfBytes;
    static constexpr int kStageBytes = al(sVsf + kVsfBytes);
    static constexpr int oP = oStage + kStages * kStageBytes;    // 2 buffers
    static constexpr int oPsf = oP + 2 * kPBytes;                 // 2 x 1024
    static constexpr int oLut = oPsf + 2 * kPsfBytes;            // 256 x {log2(2^pre/s), s, 2^pre/s, 0}
    static constexpr int oM = oLut + 4096;                       // running max [2][128]
    static constexpr int oAlpha = oM + 1024;                     // alpha ring [4][128]
    static constexpr int oL = oAlpha + 2048;                     // per warpgroup {l, m} [2][2][128]
    static constexpr int oBar = oL + 2048;
    static constexpr int kSmemBytes = oBar + 512 + 1024;
    // TMEM columns
    static constexpr uint32_t tS = 0;                  // S_A at 0, S_B at 128
    static constexpr uint32_t tO = 256;
    static constexpr uint32_t tSfq = 256 + D;          // 2 slots of 4 * (D / 64)
    static constexpr uint32_t tSfk = tSfq + 8 * (D / 64);
    static constexpr uint32_t tSfp = tSfk + 4 * (D / 64);
    static constexpr uint32_t tSfv = tSfp + 8;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(tSfv + 8 <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Barrier slots (uint64 each) after oBar.  Counts: "commit" = one
// tcgen05.commit arrival; "128" = every thread of one warpgroup.
enum : int {
    kBarQFull = 0,     // 2: Q tile slot loaded (transaction bytes)
    kBarQEmpty = 2,    // 2: commit after the tile's last S product
    kBarSFull = 4,     // 2: commit: S_X holds block g
    kBarPFull = 6,     // 2: 128: warpgroup X has read S_X and written P_X
    kBarPFree = 8,     // 2: commit: the P V product reading P_X is done
    kBarPvDone = 10,   // 1: commit after every P V product, in order
    kBarOReady = 11,   // 1: 128: O rescaled (or free) for the next P V
    kBarMFull = 12,    // 2: 128: running max of block g in slot g%2
    kBarAlpha = 14,    // 4: 128: alpha of block g in slot g%4
    kBarLFull = 18,    // 2: 128: warpgroup X's {l, m} for the tile
    kBarLFree = 20,    // 2: 128: the correction warps have read them
    kBarDrain = 22,    // 1: commit: every tcgen05 op has completed
    kBarSEmpty = 23,   // 2: 128: warpgroup X has loaded all of S_X
    kBarKv = 25        // kStages full, then kStages empty (commit)
};

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

// Bounded wait that ignores the abort flag (used to drain copies and MMAs
// in flight before the CTA exits).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kWaitLimitNs) {
            atomicOr(&g_sa3_status, 1u);
            return;
        }
    }
}

// Static list of work for CTA `c` of `G`, returned one 128-row Q tile at a
// time.  A work unit is one Q tile, or with the causal mask a pair of tiles
// (rank r and its mirror nqt-1-r, heavier first), so that all units cost
// about the same (t + 1 blocks for tile t, nqt + 1 for a pair); with an odd
// tile count each head's middle tile is a unit of its own, and these come
// last, after every pair, where they fill the last round.  Pairs and tiles
// are grouped by `hg` heads, so that the CTAs working at one time share
// the K / V of a few heads in L2; inside a group they run rank by rank.
// CTA c takes the units c, then 2G-1-c, then 2G+c, ... (alternating
// direction evens out what differences remain).
struct Sched {
    int c, G, k, total, per, grouped, BH, nqt, nkvt, hg, off, causal;
    int pend_bh, pend_tile;  // the second tile of the current pair, if any
    bool pend;
    __host__ __device__ void init(const AttnParams &p, int cta, int ctas) {
        c = cta;
        G = ctas;
        k = 0;
        BH = p.BH;
        nqt = p.Npq / kBlk;
        nkvt = p.Np / kBlk;
        hg = p.hg;
        off = p.N - p.Nq;
        causal = p.causal;
        per = grouped_per_head(nqt, causal);
        grouped = BH * per;
        total = grouped + ((causal && (nqt & 1)) ? BH : 0);
        pend = false;
    }
    // grouped units per head: pairs (causal) or tiles; plus, causal with an
    // odd tile count, one middle tile per head after all of them
    __host__ __device__ static int grouped_per_head(int nqt, int causal) { return causal ? nqt / 2 : nqt; }
    __host__ __device__ static long long units(int BH, int nqt, int causal) {
        return static_cast<long long>(BH) * grouped_per_head(nqt, causal) + ((causal && (nqt & 1)) ? BH : 0);
    }
    // KV blocks that tile t processes: up to the last key any of its rows
    // sees (0: none)
    __host__ __device__ int blocks_of(int tile) const {
        if (!causal) return nkvt;
        const int last = tile * kBlk + kBlk - 1 + off;
        const int nb = last < 0 ? 0 : last / kBlk + 1;
        return nb < nkvt ? nb : nkvt;
    }
    __host__ __device__ bool next(int &bh, int &tile, int &n) {
        if (pend) {
            pend = false;
            bh = pend_bh;
            tile = pend_tile;
            n = blocks_of(tile);
            return true;
        }
        while (true) {
            const int start = k * G;
            if (start >= total) return false;
            const int pos = start + ((k & 1) ? G - 1 - c : c);
            ++k;
            if (pos >= total) continue;  // last round: this CTA's slot is past the end
            if (pos >= grouped) {
                bh = pos - grouped;  // a middle tile (causal, odd tile count)
                tile = nqt >> 1;
                n = blocks_of(tile);
                return true;
            }
            const int gsz = hg * per;
            const int full = BH / hg;
            int grp, idx, h;
            if (pos < full * gsz) {
                grp = pos / gsz;
                idx = pos - grp * gsz;
                h = hg;
            } else {
                grp = full;
                idx = pos - full * gsz;
                h = BH - full * hg;
            }
            const int rank = idx / h;
            bh = grp * hg + (idx - rank * h);
            if (causal) {
                tile = nqt - 1 - rank;
                if (rank != tile) {
                    pend = true;
                    pend_bh = bh;
                    pend_tile = rank;
                }
            } else {
                tile = rank;
            }
            n = blocks_of(tile);
            return true;
        }
    }
};

// kCross: query and key/value lengths differ (bottom-right causal offset,
// rows that may see no key).  kTwo: P is pre-scaled by 2^11 before it is
// microscaled (two-level P).  Each term is compiled only into the instances
// that use it.
template <int D, bool kCross, bool kTwo>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using C = Cfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_s - raw_s);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + C::oBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kBarKv + 2 * S);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint64_t *kv_full = bars + kBarKv;
    uint64_t *kv_empty = bars + kBarKv + S;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars + kBarQFull + i, 1);
            mbar_init(bars + kBarQEmpty + i, 1);
            mbar_init(bars + kBarSFull + i, 1);
            mbar_init(bars + kBarPFull + i, 128);
            mbar_init(bars + kBarSEmpty + i, 128);
            mbar_init(bars + kBarPFree + i, 1);
            mbar_init(bars + kBarMFull + i, 128);
            mbar_init(bars + kBarLFull + i, 128);
            mbar_init(bars + kBarLFree + i, 128);
        }
        for (int i = 0; i < 4; ++i) mbar_init(bars + kBarAlpha + i, 128);
        mbar_init(bars + kBarPvDone, 1);
        mbar_init(bars + kBarOReady, 128);
        mbar_init(bars + kBarDrain, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(kv_full + s, 1);
            mbar_init(kv_empty + s, 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < 256) {
        // per E4M3 scale code s: {log2(2^pre / s), s, fp32(1 / s) * 2^pre}
        // (pre = 11 under kTwo, else 0).  Code 0 (and the NaN codes, which
        // the saturating conversion never produces) map to {pre, 1, 0}: such
        // a block holds only P < 6 * 2^-10 (times 2^pre), whose codes are 0
        // at scale 1 exactly as at scale 0 (and 1/s = 0 makes them 0 too),
        // and whose row-sum terms stay P.
        const float v = e4m3_value(threadIdx.x);
        const bool unit = v == 0.0f || v != v;
        const float pre = kTwo ? 11.0f : 0.0f;
        const float sc = kTwo ? 2048.0f : 1.0f;
        reinterpret_cast<float4 *>(base + C::oLut)[threadIdx.x] =
            unit ? make_float4(pre, 1.0f, 0.0f, 0.0f) : make_float4(pre - log2f(v), v, __frcp_rn(v) * sc, 0.0f);
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nqt = p.Npq / kBlk;
    const int nkvt = p.Np / kBlk;

    if (warp == kWarpProducer) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            Sched sc;
            sc.init(p, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
            int bh, tile, n;
            int t = 0;    // tiles with at least one block (Q slot = t % 2)
            int g = 0;    // KV blocks issued
            bool ok = true;
            while (ok && sc.next(bh, tile, n)) {
                if (n == 0) continue;
                const int qs = t & 1;
                if (t >= 2 && !mbar_wait(bars + kBarQEmpty + qs, ((t >> 1) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                uint64_t *bq = bars + kBarQFull + qs;
                mbar_arrive_expect_tx(bq, C::kQBytes + C::kSfBytes);
                tma_load_2d(base + C::oQ + qs * C::kQSlot, &tm_q, 0, bh * p.Npq + tile * kBlk, bq);
                bulk_load(base + C::oQsf + qs * C::kSfBytes,
                          p.q_sf + static_cast<size_t>(bh * nqt + tile) * C::kSfBytes, C::kSfBytes, bq);
                ++t;
                for (int j = 0; j < n; ++j, ++g) {
                    const int s = g % S;
                    if (g >= S && !mbar_wait(kv_empty + s, ((g / S) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = base + C::oStage + s * C::kStageBytes;
                    uint64_t *bf = kv_full + s;
                    mbar_arrive_expect_tx(bf, C::kQBytes + C::kSfBytes + C::kVBytes + C::kVsfBytes);
                    tma_load_2d(st + C::sK, &tm_k, 0, bh * p.Np + j * kBlk, bf);
                    bulk_load(st + C::sKsf, p.k_sf + static_cast<size_t>(bh * nkvt + j) * C::kSfBytes,
                              C::kSfBytes, bf);
                    tma_load_2d(st + C::sV, &tm_v, j * 64, bh * D, bf);
                    bulk_load(st + C::sVsf, p.vt_sf + (static_cast<size_t>(bh) * (p.Np / 64) + 2 * j) * 512,
                              C::kVsfBytes, bf);
                }
            }
            // Let every copy this thread started land before the CTA exits.
            for (int i = t - 2 < 0 ? 0 : t - 2; i < t; ++i) drain_wait(bars + kBarQFull + (i & 1), (i >> 1) & 1);
            for (int i = g - S < 0 ? 0 : g - S; i < g; ++i) drain_wait(kv_full + i % S, (i / S) & 1);
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // --------------------------------------------------------------- MMA
        if (lane == 0) {
            // descriptors from precomputed low words (address >> 4 | leading
            // offset << 16) and a per-operand-kind high word
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
            const uint32_t q_lo0 = lo_of(base_s + C::oQ, 1), qsf_lo0 = lo_of(base_s + C::oQsf, 8);
            const uint32_t p_lo0 = lo_of(base_s + C::oP, 1), psf_lo0 = lo_of(base_s + C::oPsf, 8);
            constexpr uint32_t kQLo = static_cast<uint32_t>(C::kQSlot) >> 4;
            constexpr uint32_t kQsfLo = static_cast<uint32_t>(C::kSfBytes) >> 4;

            // Two cursors over the same block sequence: `qk` runs up to two
            // blocks ahead of `pv`.
            struct Cursor {
                Sched sc;
                int bh, tile, n, j, t, g;  // t: index of the tile among those with blocks
                bool valid;
                __device__ void start(const AttnParams &pp) {
                    sc.init(pp, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
                    t = -1;
                    g = -1;
                    j = 0;
                    n = 0;
                    valid = true;
                    advance();
                }
                __device__ void advance() {
                    ++g;
                    if (++j < n) return;
                    j = 0;
                    while (true) {
                        if (!sc.next(bh, tile, n)) {
                            valid = false;
                            return;
                        }
                        if (n > 0) break;
                    }
                    ++t;
                }
            };
            Cursor qk, pv;
            qk.start(p);
            pv.start(p);
            bool ok = true;
            auto issue_qk = [&]() -> bool {
                const int g = qk.g, s = g % S, x = g & 1, qs = qk.t & 1;
                if (qk.j == 0) {
                    if (!mbar_wait(bars + kBarQFull + qs, (qk.t >> 1) & 1, abort_flag)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int a = 0; a < D / 64; ++a)
                        tc_cp_32x128b_warpx4(tmem + C::tSfq + (4 * (D / 64)) * qs + 4 * a,
                                             desc(qsf_lo0 + qs * kQsfLo + 32 * a, kHiSF));
                }
                if (!mbar_wait(kv_full + s, (g / S) & 1, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int a = 0; a < D / 64; ++a)
                    tc_cp_32x128b_warpx4(tmem + C::tSfk + 4 * a, desc(ksf_lo0 + s * kStageLo + 32 * a, kHiSF));
                const uint32_t qa = q_lo0 + qs * kQLo;
                const uint32_t kb = k_lo0 + s * kStageLo;
                const uint32_t sfq = tmem + C::tSfq + (4 * (D / 64)) * qs;
#pragma unroll
                for (int kc = 0; kc < D / 64; ++kc)
                    tc_mma_mxf4nvf4(tmem + C::tS + 128 * x, desc(qa + 2 * kc, kHiQK), desc(kb + 2 * kc, kHiQK),
                                    idesc_qk, sfq + 4 * kc, tmem + C::tSfk + 4 * kc, kc > 0);
                tc_commit(bars + kBarSFull + x);
                if (qk.j == qk.n - 1) tc_commit(bars + kBarQEmpty + qs);
                qk.advance();
                return true;
            };
            // prologue: the first two S products (S_A and S_B start free)
            for (int i = 0; i < 2 && ok && qk.valid; ++i) ok = issue_qk();
            while (ok && pv.valid) {
                const int g = pv.g, s = g % S, x = g & 1;
                if (qk.valid) {
                    // warpgroup x has loaded S_x of block g: block g + 2 may go there
                    if (!mbar_wait(bars + kBarSEmpty + x, (g >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!(ok = issue_qk())) break;
                }
                // warpgroup x has written P_x for block g
                if (!mbar_wait(bars + kBarPFull + x, (g >> 1) & 1, abort_flag) ||
                    !mbar_wait(bars + kBarOReady, g & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t psf = psf_lo0 + x * (C::kPsfBytes >> 4);
                const uint32_t vsf = vsf_lo0 + s * kStageLo;
                tc_cp_32x128b_warpx4(tmem + C::tSfp, desc(psf, kHiSF));
                tc_cp_32x128b_warpx4(tmem + C::tSfp + 4, desc(psf + 32, kHiSF));
                tc_cp_32x128b_warpx4(tmem + C::tSfv, desc(vsf, kHiSF));
                tc_cp_32x128b_warpx4(tmem + C::tSfv + 4, desc(vsf + 32, kHiSF));
                const uint32_t pa = p_lo0 + x * (C::kPBytes >> 4);
                const uint32_t vb = v_lo0 + s * kStageLo;
#pragma unroll
                for (int kc = 0; kc < 2; ++kc)
                    tc_mma_mxf4nvf4(tmem + C::tO, desc(pa + 2 * kc, kHiPV), desc(vb + 2 * kc, kHiPV), idesc_pv,
                                    tmem + C::tSfp + 4 * kc, tmem + C::tSfv + 4 * kc, (pv.j > 0 || kc > 0) ? 1u : 0u);
                tc_commit(bars + kBarPFree + x);
                tc_commit(bars + kBarPvDone);
                tc_commit(kv_empty + s);
                pv.advance();
            }
            // Every tcgen05 op issued above completes before TMEM is freed.
            tc_commit(bars + kBarDrain);
            drain_wait(bars + kBarDrain, 0);
        }
        __syncwarp();
    } else if (warp < kWarpCorr) {
        // ----------------------------------------------------------- softmax
        const int X = warp >> 2;           // warpgroup: blocks with g % 2 == X
        const int wq = warp & 3;           // TMEM lane quadrant = rows 32*wq ..
        const int r = wq * 32 + lane;      // row inside the tile
        const float c2 = p.scale_log2;
        const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16) + C::tS + 128 * X;
        uint8_t *P = base + C::oP + X * C::kPBytes;
        uint8_t *Psf = base + C::oPsf + X * C::kPsfBytes;
        float *mrow = reinterpret_cast<float *>(base + C::oM);
        float *arow = reinterpret_cast<float *>(base + C::oAlpha);
        float *lrow = reinterpret_cast<float *>(base + C::oL) + X * 256;
        const float4 *lut = reinterpret_cast<const float4 *>(base + C::oLut);
        Sched sc;
        sc.init(p, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
        int bh, tile, n;
        int g0 = 0;       // first block of the current tile
        int mine = 0;     // blocks this warpgroup has processed
        int tiles = 0;    // tiles in which this warpgroup processed a block
        bool ok = true;
        while (ok && sc.next(bh, tile, n)) {
            const int grow = tile * kBlk + r;
            float m_x = -INFINITY, l_x = 0.0f;  // this warpgroup's share of the row sum, relative to m_x
            bool any = false;
            for (int j = X ^ (g0 & 1); j < n; j += 2) {
                const int g = g0 + j;
                if (!warp_wait(bars + kBarSFull + X, mine & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // columns col0 + k with k >= lim are masked for this row
                const int col0 = j * kBlk;
                int lim = kBlk;
                if (col0 + kBlk > p.N) lim = p.N - col0;
                if (p.causal) lim = min(lim, grow + sc.off - col0 + 1);
                const bool masked = __any_sync(0xffffffffu, lim < kBlk);
                // pass 1: the maxima of the eight 16-column blocks; the loads
                // of later 32-column chunks overlap the maxima of earlier ones
                float bm[8];
                auto block_max = [&](uint32_t(&x32)[32], int q) {
                    if (masked) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (32 * q + e >= lim) x32[e] = __float_as_uint(-INFINITY);
                    }
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        const uint32_t *x = &x32[16 * hb];
                        const float m0 = max3f(__uint_as_float(x[0]), __uint_as_float(x[1]), __uint_as_float(x[2]));
                        const float m1 = max3f(__uint_as_float(x[3]), __uint_as_float(x[4]), __uint_as_float(x[5]));
                        const float m2 = max3f(__uint_as_float(x[6]), __uint_as_float(x[7]), __uint_as_float(x[8]));
                        const float m3 = max3f(__uint_as_float(x[9]), __uint_as_float(x[10]), __uint_as_float(x[11]));
                        const float m4 = max3f(__uint_as_float(x[12]), __uint_as_float(x[13]), __uint_as_float(x[14]));
                        bm[2 * q + hb] = max3f(max3f(m0, m1, m2), max3f(m3, m4, __uint_as_float(x[15])), m0);
                    }
                };
                {
                    uint32_t c0[32], c1[32], c2[32];
                    tmem_ld32(trow, c0);
                    tmem_ld32(trow + 32, c1);
                    tmem_ld_wait();
                    reg_fence32(c0);
                    reg_fence32(c1);
                    tmem_ld32(trow + 64, c2);
                    block_max(c0, 0);
                    block_max(c1, 1);
                    tmem_ld_wait();
                    reg_fence32(c2);
                    tmem_ld32(trow + 96, c0);
                    block_max(c2, 2);
                    tmem_ld_wait();
                    reg_fence32(c0);
                    block_max(c0, 3);
                }
                const float rmax = max3f(max3f(bm[0], bm[1], bm[2]), max3f(bm[3], bm[4], bm[5]), fmaxf(bm[6], bm[7]));
                // running max of block g-1 (waited for even at a tile's first
                // block, which keeps the slots of the exchange in order)
                float m_prev = -INFINITY;
                if (g > 0) {
                    if (!warp_wait(bars + kBarMFull + ((g - 1) & 1), ((g - 1) >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (j > 0) m_prev = mrow[((g - 1) & 1) * kBlk + r];
                }
                // (kCross) clamped below at -FLT_MAX: a row that has seen no
                // key yet gets P = 0 and alpha = 0, never inf - inf
                const float m_new = kCross ? fmaxf(fmaxf(m_prev, __fmul_rn(rmax, c2)), -3.402823466e38f)
                                           : fmaxf(m_prev, __fmul_rn(rmax, c2));
                mrow[(g & 1) * kBlk + r] = m_new;
                mbar_arrive(bars + kBarMFull + (g & 1));
                arow[(g & 3) * kBlk + r] = ex2(__fsub_rn(m_prev, m_new));
                mbar_arrive(bars + kBarAlpha + (g & 3));
                const float nm = -m_new;
                // block scales: s_b = E4M3(amax_b / 6), amax_b = 2^(bm_b*c - m'),
                // two blocks per conversion (byte 0: block b)
                uint32_t scw[2];
#pragma unroll
                for (int b = 0; b < 8; b += 2) {
                    const float a0 = ex2(__fadd_rn(__fmul_rn(bm[b], c2), nm));
                    const float a1 = ex2(__fadd_rn(__fmul_rn(bm[b + 1], c2), nm));
                    // amax' / 6 with amax' = 2^11 * amax under kTwo (exact: 2^11 * fp32(1/6))
                    constexpr float kDiv = kTwo ? 2048.0f * kSixth : kSixth;
                    const uint32_t sc2 = cvt_e4m3x2(a1 * kDiv, a0 * kDiv);
                    if ((b & 2) == 0) scw[b >> 2] = sc2;
                    else scw[b >> 2] |= sc2 << 16;
                }
                // P_X is free once the P V product of this warpgroup's
                // previous block has completed (long before, normally)
                if (mine > 0 && !warp_wait(bars + kBarPFree + X, (mine - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t *prow = P + (r >> 3) * 512 + (r & 7) * 64;
                const int sw = (r & 7) >> 1;
                // pass 2: the recipe's own steps, 32 columns (one 16-byte
                // chunk of the P row) at a time: t = fp32(S*c), u = t - m'
                // (exact near the row maximum, whose P is then exactly 1),
                // P = 2^u, y = fp32(P * (1/s_b)) and its E2M1 codes, and the
                // row sum of the unquantized P.  A peaked row's output is then
                // the recipe's own fp32 value, not one rounding away from it:
                // its bf16 results often sit on rounding ties, which an ulp of
                // l would decide the other way.  Under kTwo y and the row sum
                // carry 2^11 (l and O both do).  The loop over chunk pairs is
                // kept rolled: the softmax code must stay small enough for the
                // instruction cache shared with the other roles' warps.
                const uint64_t cc = pack2(c2, c2);
                const uint64_t nn = pack2(nm, nm);
                const uint64_t sc8 = static_cast<uint64_t>(scw[0]) | (static_cast<uint64_t>(scw[1]) << 32);
                float sum = 0.0f;
                auto chunk = [&](uint32_t(&x32)[32], int q) {
                    if (masked) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (32 * q + e >= lim) x32[e] = __float_as_uint(-INFINITY);
                    }
                    uint32_t pc[4];
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        const int b = 2 * q + hb;
                        const uint32_t *x = &x32[16 * hb];
                        const float r_b = lut[(sc8 >> (8 * b)) & 0xFF].z;  // 2^pre / s_b
                        const uint64_t rr = pack2(r_b, r_b);
                        uint64_t pp[8], vy[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint64_t t2 = mul2(pack2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), cc);
                            const uint64_t u2 = add2(t2, nn);
                            pp[e] = pack2(ex2(lo2(u2)), ex2(hi2(u2)));
                            vy[e] = mul2(pp[e], rr);
                        }
                        const uint64_t s01 = add2(add2(pp[0], pp[1]), add2(pp[2], pp[3]));
                        const uint64_t s23 = add2(add2(pp[4], pp[5]), add2(pp[6], pp[7]));
                        const uint64_t sb = add2(s01, s23);
                        sum += lo2(sb) + hi2(sb);
                        pc[2 * hb] = cvt_e2m1x8(lo2(vy[0]), hi2(vy[0]), lo2(vy[1]), hi2(vy[1]), lo2(vy[2]),
                                                hi2(vy[2]), lo2(vy[3]), hi2(vy[3]));
                        pc[2 * hb + 1] = cvt_e2m1x8(lo2(vy[4]), hi2(vy[4]), lo2(vy[5]), hi2(vy[5]), lo2(vy[6]),
                                                    hi2(vy[6]), lo2(vy[7]), hi2(vy[7]));
                    }
                    *reinterpret_cast<uint4 *>(prow + ((q ^ sw) << 4)) = make_uint4(pc[0], pc[1], pc[2], pc[3]);
                };
                uint32_t sa[32], sb2[32];
                tmem_ld32(trow, sa);
                tmem_ld_wait();
                reg_fence32(sa);
#pragma unroll 1
                for (int qq = 0; qq < 2; ++qq) {
                    tmem_ld32(trow + 64 * qq + 32, sb2);
                    chunk(sa, 2 * qq);
                    tmem_ld_wait();
                    reg_fence32(sb2);
                    if (qq == 0) {
                        tmem_ld32(trow + 64, sa);
                    } else {
                        // all of S_X is in registers: the MMA may overwrite it
                        tc_fence_before();
                        mbar_arrive(bars + kBarSEmpty + X);
                    }
                    chunk(sb2, 2 * qq + 1);
                    if (qq == 0) {
                        tmem_ld_wait();
                        reg_fence32(sa);
                    }
                }
                // blocks 4a .. 4a+3 = the four columns of scale atom a
#pragma unroll
                for (int a = 0; a < 2; ++a)
                    *reinterpret_cast<uint32_t *>(Psf + 512 * a + 16 * (r & 31) + 4 * (r >> 5)) = scw[a];
                if (kTwo) sum *= 2048.0f;  // l carries 2^11 like O (exact)
                // this warpgroup's share of the row sum, relative to m'
                l_x = any ? fmaf(l_x, ex2(__fsub_rn(m_x, m_new)), sum) : sum;
                m_x = m_new;
                any = true;
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bars + kBarPFull + X);
                ++mine;
            }
            if (!ok) break;
            if (any) {
                // this warpgroup's {l, m} of the tile for the epilogue
                if (tiles > 0 && !warp_wait(bars + kBarLFree + X, (tiles - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                lrow[r] = l_x;
                lrow[kBlk + r] = m_x;
                mbar_arrive(bars + kBarLFull + X);
                ++tiles;
            }
            g0 += n;
        }
    } else {
        // -------------------------------------------------------- correction
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16) + C::tO;
        const float *arow = reinterpret_cast<const float *>(base + C::oAlpha);
        const float *lrow = reinterpret_cast<const float *>(base + C::oL);
        Sched sc;
        sc.init(p, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
        int bh, tile, n;
        int g0 = 0;
        int tiles[2] = {0, 0};  // tiles in which warpgroup A / B took part
        bool ok = true;
        while (ok && sc.next(bh, tile, n)) {
            const int grow = tile * kBlk + r;
            __nv_bfloat16 *orow = p.out + (static_cast<size_t>(bh) * p.Nq + grow) * D;
            if (kCross && n == 0) {
                // causal with more queries than keys: no row of this tile sees a key
                if (grow < p.Nq) {
#pragma unroll
                    for (int v = 0; v < D / 8; ++v) reinterpret_cast<uint4 *>(orow)[v] = make_uint4(0u, 0u, 0u, 0u);
                }
                continue;
            }
            for (int j = 0; j < n; ++j) {
                const int g = g0 + j;
                if (!warp_wait(bars + kBarAlpha + (g & 3), (g >> 2) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const float a = arow[(g & 3) * kBlk + r];
                // P V of block g-1 must be done before O may be rescaled.  Its
                // completion is waited for at every block, rescaled or not:
                // the waits on kBarPvDone then take its phases one by one,
                // in order (a parity wait can tell apart only the current
                // phase and the one before)
                if (j > 0) {
                    if (!warp_wait(bars + kBarPvDone, (g - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                if (j > 0 && __any_sync(0xffffffffu, a != 1.0f)) {
                    // O = alpha * O for this warp's 32 rows
                    const uint64_t aa = pack2(a, a);
                    // two 32-column chunks per TMEM round trip
#pragma unroll
                    for (int q = 0; q < D / 32; q += 2) {
                        uint32_t o0[32], o1[32];
                        tmem_ld32(trow + 32 * q, o0);
                        tmem_ld32(trow + 32 * q + 32, o1);
                        tmem_ld_wait();
                        reg_fence32(o0);
                        reg_fence32(o1);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const uint64_t v0 = mul2(pack2(__uint_as_float(o0[e]), __uint_as_float(o0[e + 1])), aa);
                            o0[e] = __float_as_uint(lo2(v0));
                            o0[e + 1] = __float_as_uint(hi2(v0));
                            const uint64_t v1 = mul2(pack2(__uint_as_float(o1[e]), __uint_as_float(o1[e + 1])), aa);
                            o1[e] = __float_as_uint(lo2(v1));
                            o1[e + 1] = __float_as_uint(hi2(v1));
                        }
                        tmem_st32(trow + 32 * q, o0);
                        tmem_st32(trow + 32 * q + 32, o1);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(bars + kBarOReady);
            }
            if (!ok) break;
            // epilogue: wait for the tile's last P V, combine the two
            // warpgroups' row sums, out = bf16(O / l) for rows < Nq
            const int glast = g0 + n - 1;
            if (!warp_wait(bars + kBarPvDone, glast & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float lx[2], mx[2];
            bool part[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                part[x] = n >= 2 || (g0 & 1) == x;
                lx[x] = 0.0f;
                mx[x] = -INFINITY;
                if (part[x]) {
                    if (!warp_wait(bars + kBarLFull + x, tiles[x] & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    lx[x] = lrow[x * 256 + r];
                    mx[x] = lrow[x * 256 + kBlk + r];
                    mbar_arrive(bars + kBarLFree + x);
                    ++tiles[x];
                }
            }
            if (!ok) break;
            const float mf = fmaxf(mx[0], mx[1]);
            float l = 0.0f;
#pragma unroll
            for (int x = 0; x < 2; ++x)
                if (part[x]) l = fmaf(lx[x], mx[x] == mf ? 1.0f : ex2(__fsub_rn(mx[x], mf)), l);
            // a row that sees no key (kCross only) outputs 0
            const float inv = (!kCross || l > 0.0f) ? __frcp_rn(l) : 0.0f;
            // O is read chunk by chunk; the next tile's first P V may
            // overwrite it only after this warpgroup's next OReady arrival,
            // which follows in program order
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(trow + 32 * q, o);
                tmem_ld_wait();
                reg_fence32(o);
                uint32_t w[16];
                if (p.v_mean) {
                    // V smoothing: the mean of V comes back after O / l (a row
                    // that sees no key stays 0)
                    const float4 *vm = reinterpret_cast<const float4 *>(p.v_mean + static_cast<size_t>(bh) * D + 32 * q);
                    const bool live = !kCross || l > 0.0f;
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
                if (grow < p.Nq) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * q);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
            tc_fence_before();
            g0 += n;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// Host: CTAs of the persistent grid (one per SM, at most one per tile) and
// heads per group of the work list (enough tiles for about two rounds).
inline int persistent_grid(const AttnParams &p, int nsm) {
    const long long units = Sched::units(p.BH, p.Npq / kBlk, p.causal);
    return static_cast<int>(units < nsm ? units : nsm);
}
inline int heads_per_group(const AttnParams &p, int grid) {
    const int per = Sched::grouped_per_head(p.Npq / kBlk, p.causal);
    if (per == 0) return 1;
    const int hg = (2 * grid + per - 1) / per;
    return hg < 1 ? 1 : (hg > p.BH ? p.BH : hg);
}

template <int D>
cudaError_t launch_d(const AttnParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t stream) {
    using C = Cfg<D>;
    const bool cross = p.Nq != p.N;
    const bool two = p.p_pre_log2 != 0.0f;
    auto kernel = cross ? (two ? attn_fwd_kernel<D, true, true> : attn_fwd_kernel<D, true, false>)
                        : (two ? attn_fwd_kernel<D, false, true> : attn_fwd_kernel<D, false, false>);
    cudaError_t e = cross ? (two ? smem_attr_once<attn_fwd_kernel<D, true, true>>(C::kSmemBytes)
                                 : smem_attr_once<attn_fwd_kernel<D, true, false>>(C::kSmemBytes))
                          : (two ? smem_attr_once<attn_fwd_kernel<D, false, true>>(C::kSmemBytes)
                                 : smem_attr_once<attn_fwd_kernel<D, false, false>>(C::kSmemBytes));
    if (e != cudaSuccess) return e;
    AttnParams q = p;
    const int grid = persistent_grid(p, sm_count());
    q.hg = heads_per_group(p, grid);
    kernel<<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, q);
    return cudaGetLastError();
}

}  // namespace attn

inline cudaError_t launch_attn(const AttnParams &p, const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                               const CUtensorMap &tm_v, int d, cudaStream_t stream) {
    return d == 128 ? attn::launch_d<128>(p, tm_q, tm_k, tm_v, stream)
                    : attn::launch_d<64>(p, tm_q, tm_k, tm_v, stream);
}

}  // namespace sa3
