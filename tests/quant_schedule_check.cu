// Host-side check of the quantizer's static schedule (SchedA in quant.cuh),
// run by tests/test_quant_schedule.py: for every listed shape and grid size,
// with and without V smoothing, each Q tile and V tile is handed out
// exactly once (V tiles: none with V smoothing, whose V tiles go to the
// second launch), each K tile (and, with V smoothing, each V tile) exactly
// once to a column sum, every summed tile belongs to the chunk it is
// reported in, every chunk is flushed exactly once (its last tile), no job
// is out of range, and no CTA receives more than the average plus one chunk
// of tiles; the thread -> (row, channel half) map of a Q/K tile is one to
// one.  Only host code runs.
#include "quant.cuh"

#include <cstdio>
#include <vector>

int main() {
    {
        // the thread -> (row, channel half) map of a Q/K tile: one to one,
        // and the 8 threads of each shared-memory phase on 8 row classes
        std::vector<int> seen(256, 0);
        for (int t = 0; t < 256; ++t) {
            const int r = sa3::quant::qk_row(t), h = sa3::quant::qk_part(t);
            if (r < 0 || r >= 128 || h < 0 || h > 1 || seen[2 * r + h]++ ||
                h != sa3::quant::qk_part(t & ~7) || (r & 7) != (t & 7)) {
                printf("qk_row / qk_part: bad map at thread %d\n", t);
                return 1;
            }
        }
    }
    long long checked = 0;
    for (int BH : {1, 2, 3, 7, 30, 32, 128, 151})
        for (int N : {1, 100, 128, 129, 300, 1000, 4096, 8192, 17776, 32768})
            for (int Nq : {N, 1, 77, 2000}) {
                const int ntile = (N + 127) / 128;
                const int ntq = (Nq + 127) / 128;
                const int chunk = 512 * (((N + 511) / 512 + 15) / 16);  // sa3_kmean_chunk
                const int nchunk = (N + chunk - 1) / chunk;
                const int tpc = chunk / 128;
                for (int vs = 0; vs < 2; ++vs)
                for (int G : {1, 2, 5, 37, 148, 296}) {
                    const long long work = (long long)BH * (ntq + (vs ? 0 : ntile)) + (long long)BH * nchunk * (vs ? 2 : 1);
                    const int Gx = work < G ? (int)work : G;
                    std::vector<int> q(BH * ntq, 0), v(BH * ntile, 0), k(BH * ntile, 0), last(BH * nchunk, 0);
                    std::vector<int> vsum(BH * ntile, 0), vlast(BH * nchunk, 0);
                    int maxload = 0;
                    for (int g = 0; g < Gx; ++g) {
                        sa3::quant::SchedA s;
                        s.init(BH, ntq, ntile, nchunk, tpc, g, Gx, vs != 0);
                        sa3::quant::TileJob t;
                        int load = 0;
                        while (s.next(t)) {
                            ++load;
                            if (t.bh < 0 || t.bh >= BH || t.tile < 0 || t.tile >= (t.kind == 0 ? ntq : ntile)) {
                                printf("job out of range: BH=%d N=%d Nq=%d G=%d\n", BH, N, Nq, Gx);
                                return 1;
                            }
                            if (t.kind == 0) {
                                q[t.bh * ntq + t.tile]++;
                            } else if (t.kind == 1) {
                                v[t.bh * ntile + t.tile]++;
                            } else {
                                (t.kind == 2 ? k : vsum)[t.bh * ntile + t.tile]++;
                                if (t.tile / tpc != t.chunk) {
                                    printf("summed tile outside its chunk: BH=%d N=%d G=%d\n", BH, N, Gx);
                                    return 1;
                                }
                                if (t.last) (t.kind == 2 ? last : vlast)[t.bh * nchunk + t.chunk]++;
                            }
                        }
                        if (load > maxload) maxload = load;
                    }
                    for (int i = 0; i < BH * ntq; ++i)
                        if (q[i] != 1) {
                            printf("Q tile %d handed out %d times: BH=%d Nq=%d G=%d\n", i, q[i], BH, Nq, Gx);
                            return 1;
                        }
                    for (int i = 0; i < BH * ntile; ++i)
                        if (v[i] != (vs ? 0 : 1) || k[i] != 1 || vsum[i] != (vs ? 1 : 0)) {
                            printf("V/K tile %d: %d / %d / %d times: BH=%d N=%d G=%d vs=%d\n", i, v[i], k[i], vsum[i],
                                   BH, N, Gx, vs);
                            return 1;
                        }
                    for (int i = 0; i < BH * nchunk; ++i)
                        if (last[i] != 1 || vlast[i] != (vs ? 1 : 0)) {
                            printf("chunk %d flushed %d / %d times: BH=%d N=%d G=%d\n", i, last[i], vlast[i], BH, N, Gx);
                            return 1;
                        }
                    const double avg = (double)((long long)BH * ((vs ? 3LL : 2LL) * ntile + ntq)) / Gx;
                    if (Gx > 2 && maxload > avg + tpc + 2) {
                        printf("imbalance: BH=%d N=%d Nq=%d G=%d max %d avg %.1f\n", BH, N, Nq, Gx, maxload, avg);
                        return 1;
                    }
                    ++checked;
                }
            }
    printf("ok %lld cases\n", checked);
    return 0;
}
