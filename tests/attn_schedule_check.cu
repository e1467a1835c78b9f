// Host-side check of the FP4 attention kernel's persistent work list (Sched
// in attn.cuh), run by tests/test_attn_schedule.py: for every listed shape,
// mask and grid size, each (head, Q tile) unit is handed out exactly once,
// each unit's KV block count matches the mask (0 only for queries that see
// no key), and no CTA receives more KV blocks than the average plus two of
// the largest tiles (one work unit: a tile, or with the causal mask a pair
// of tiles; checked where units cost the same, i.e. unless the causal mask
// meets more queries than keys).  Only host code runs.
#include "attn.cuh"

#include <algorithm>
#include <cstdio>
#include <vector>

int main() {
    long long checked = 0;
    for (int BH : {1, 2, 3, 7, 30, 32, 128, 151, 1000})
        for (int Nkv : {1, 100, 128, 129, 300, 1000, 4096, 8192, 17776, 32768})
            for (int Nq : {Nkv, 1, 77, 2000})
                for (int causal : {0, 1})
                    for (int nsm : {1, 5, 37, 148}) {
                        sa3::AttnParams p = {};
                        p.BH = BH;
                        p.N = Nkv;
                        p.Nq = Nq;
                        p.Np = (Nkv + 127) / 128 * 128;
                        p.Npq = (Nq + 127) / 128 * 128;
                        p.causal = causal;
                        const int G = sa3::attn::persistent_grid(p, nsm);
                        p.hg = sa3::attn::heads_per_group(p, G);
                        const int nqt = p.Npq / 128, nkvt = p.Np / 128;
                        if ((long long)BH * nqt > 200000) continue;
                        if (G > (long long)BH * nqt) {
                            printf("more CTAs than tiles\n");
                            return 1;
                        }
                        std::vector<int> seen((size_t)BH * nqt, 0);
                        std::vector<long long> load(G, 0);
                        int biggest = 0;
                        long long sum = 0;
                        for (int c = 0; c < G; ++c) {
                            sa3::attn::Sched s;
                            s.init(p, c, G);
                            int bh, tile, n;
                            while (s.next(bh, tile, n)) {
                                if (bh < 0 || bh >= BH || tile < 0 || tile >= nqt) {
                                    printf("unit out of range: BH=%d Nkv=%d Nq=%d causal=%d G=%d\n", BH, Nkv, Nq,
                                           causal, G);
                                    return 1;
                                }
                                int want = nkvt;
                                if (causal) {
                                    const int last = tile * 128 + 127 + Nkv - Nq;
                                    want = last < 0 ? 0 : std::min(nkvt, last / 128 + 1);
                                }
                                if (n != want) {
                                    printf("wrong block count: tile %d n %d want %d\n", tile, n, want);
                                    return 1;
                                }
                                seen[(size_t)bh * nqt + tile]++;
                                load[c] += n;
                                sum += n;
                                biggest = std::max(biggest, n);
                            }
                        }
                        for (size_t i = 0; i < seen.size(); ++i)
                            if (seen[i] != 1) {
                                printf("unit %zu handed out %d times: BH=%d Nkv=%d Nq=%d causal=%d G=%d\n", i,
                                       seen[i], BH, Nkv, Nq, causal, G);
                                return 1;
                            }
                        const long long mx = *std::max_element(load.begin(), load.end());
                        // (causal with more queries than keys leaves most tiles
                        // without a key: unit costs differ, only coverage is checked)
                        if ((!causal || Nq <= Nkv) && mx > (sum + G - 1) / G + 2 * biggest) {
                            printf("unbalanced: max %lld avg %lld biggest %d (BH=%d Nkv=%d Nq=%d G=%d)\n", mx,
                                   sum / G, biggest, BH, Nkv, Nq, G);
                            return 1;
                        }
                        ++checked;
                    }
    printf("ok %lld cases\n", checked);
    return 0;
}
