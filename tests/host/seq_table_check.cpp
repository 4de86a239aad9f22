// Host check of the packed-batch tile order (csrc/launch.h): for random tables of up to
// 128 sequences and every tile height, the tiles 0 .. n-1 decode to each (sequence, local
// tile) exactly once, sequence by sequence from the longest (ties in order), each
// sequence's tiles from its last (heaviest) to its first.  Prints "ok" or the first
// failure.
#include <cstdio>
#include <random>
#include <set>
#include <utility>
#include <vector>

#include "launch.h"

using tam::SeqTable;

int main() {
    std::mt19937 rng(7);
    const int heights[] = {1, 4, 8, 16, 32, 64, 128};
    for (int trial = 0; trial < 3000; ++trial) {
        SeqTable t{};
        t.n_seq = 1 + (int)(rng() % tam::kMaxSeqPerLaunch);
        t.cu[0] = 0;
        for (int s = 0; s < t.n_seq; ++s) {
            const int kind = (int)(rng() % 4);
            const int len = kind == 0 ? 0 : kind == 1 ? 1 : (int)(rng() % 900);
            t.cu[s + 1] = t.cu[s] + len;
            if (len > t.max_len) t.max_len = len;
        }
        if (t.max_len == 0) continue;
        tam::seq_table_order(t);
        for (int BQ : heights) {
            const int n = tam::seq_table_tiles(t, BQ);
            std::set<std::pair<int, int>> seen;
            int prev_s = -1, prev_L = 0, prev_len = 1 << 30;
            for (int b = 0; b < n; ++b) {
                int s, L;
                tam::seq_tile_of(t, BQ, b, s, L);
                const int len = t.cu[s + 1] - t.cu[s];
                const int nq = (len + BQ - 1) / BQ;
                if (L < 0 || L >= nq || !seen.insert({s, L}).second) {
                    std::printf("bad tile %d -> (%d, %d), trial %d BQ %d\n", b, s, L, trial, BQ);
                    return 1;
                }
                if (s != prev_s) {
                    // a new sequence starts at its last tile, no longer than the previous one,
                    // and equal lengths keep the table's order
                    if (L != nq - 1 || len > prev_len || (len == prev_len && s < prev_s)) {
                        std::printf("order broken at tile %d, trial %d BQ %d\n", b, trial, BQ);
                        return 1;
                    }
                    prev_len = len;
                } else if (L != prev_L - 1) {
                    std::printf("tiles of sequence %d out of order, trial %d\n", s, trial);
                    return 1;
                }
                prev_s = s;
                prev_L = L;
            }
            int total = 0;
            for (int s = 0; s < t.n_seq; ++s) total += (t.cu[s + 1] - t.cu[s] + BQ - 1) / BQ;
            if ((int)seen.size() != total) {
                std::printf("missing tiles, trial %d BQ %d\n", trial, BQ);
                return 1;
            }
        }
    }
    std::printf("ok\n");
    return 0;
}
