// Host-only check of the fused kernel's work schedule (compiled and run by
// tests/test_schedule_cpu.py; no GPU is touched).  For many (groups, tiles,
// blocks per tile) combinations it verifies that the pieces dealt to the groups
// cover every (tile, block) unit exactly once, that no group gets more pieces
// than the workspace provides slots for, that group loads differ by at most one
// piece plus one block per piece, and that the combine kernel's slot enumeration
// finds exactly the pieces that cover a tile.
#include <algorithm>
#include <cstdio>
#include <vector>

#include "../../discrete_diffusion_decoding_b200/csrc/dg_common.cuh"

using namespace dg;

int main() {
    int fails = 0, cases = 0;
    const int groups[] = {1, 2, 6, 13, 18, 74, 148};
    const int tiles[] = {2, 4, 6, 8, 26, 32, 64, 130, 2048};
    const int blocks[] = {1, 3, 16, 94, 256, 1031};
    for (int ng : groups)
        for (int n_pt : tiles)
            for (int T : blocks) {
                ++cases;
                std::vector<int> cover(static_cast<size_t>(n_pt) * T, 0);
                const int per = pieces_per_group(n_pt, ng);
                std::vector<std::vector<int>> slot_of_piece(n_pt);
                long long units_min = 1LL << 60, units_max = 0;
                for (int g = 0; g < ng; ++g) {
                    long long units = 0;
                    for (int j = 0; j < per + 2; ++j) {
                        int pt, tb, te;
                        if (!piece_of(g, j, ng, n_pt, T, pt, tb, te)) continue;
                        if (j >= per) { std::printf("piece beyond pieces_per_group ng=%d npt=%d T=%d\n", ng, n_pt, T); ++fails; }
                        for (int t = tb; t < te; ++t) cover[static_cast<size_t>(pt) * T + t]++;
                        units += te - tb;
                        slot_of_piece[pt].push_back(g * per + j);
                    }
                    if (units < units_min) units_min = units;
                    if (units > units_max) units_max = units;
                }
                for (size_t u = 0; u < cover.size(); ++u)
                    if (cover[u] != 1) { std::printf("unit covered %d times ng=%d npt=%d T=%d\n", cover[u], ng, n_pt, T); ++fails; break; }
                // the combine kernel's enumeration for each tile
                const int k = ranges_per_tile(n_pt, ng);
                for (int pt = 0; pt < n_pt; ++pt) {
                    std::vector<int> found;
                    for (int jj = 0; jj < k; ++jj) {
                        const int tb = static_cast<int>(static_cast<long long>(jj) * T / k);
                        const int te = static_cast<int>(static_cast<long long>(jj + 1) * T / k);
                        if (te <= tb) continue;
                        const long long pi = static_cast<long long>(jj) * n_pt + pt;
                        found.push_back(static_cast<int>(pi % ng) * per + static_cast<int>(pi / ng));
                    }
                    std::vector<int> a = found, b = slot_of_piece[pt];
                    std::sort(a.begin(), a.end());
                    std::sort(b.begin(), b.end());
                    if (a != b) { std::printf("slot mismatch ng=%d npt=%d T=%d pt=%d\n", ng, n_pt, T, pt); ++fails; break; }
                    if (static_cast<int>(a.size()) > 256) { std::printf("too many slots per tile\n"); ++fails; }
                }
                // balance: pieces per group differ by at most one and piece sizes by at most one
                // block, so group loads differ by at most one piece plus one block per piece
                const long long slack = (k == 1) ? T : (T + k - 1) / k + per;
                if (units_max - units_min > slack) {
                    std::printf("imbalance %lld ng=%d npt=%d T=%d\n", units_max - units_min, ng, n_pt, T);
                    ++fails;
                }
            }
    std::printf("schedule cases=%d fails=%d\n", cases, fails);
    return fails ? 1 : 0;
}
