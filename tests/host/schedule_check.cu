// Host-side check of the grouped GEMM's tile schedule (csrc/permute.cuh
// tile_at, csrc/moe_gemm.cuh decode_tile): for random work lists (heavy and
// light groups, ragged token counts, split-K, both GEMM modes, token bands of
// several widths) every launch position decodes to a distinct
// (group, token tile, feature block, k range), together they cover every
// tile exactly once, and each tile's rows, features and k-blocks stay inside
// its group.  For the work lists of small batches (the shared expert listed
// first, every group light), the leading tiles a launch decodes without the
// work list (decode_in_group over the shared rows: the early start of the
// gate/up launch) equal the work list's own.  Prints "OK <cases>" or the
// first violation.
#include <cstdio>
#include <random>
#include <set>
#include <tuple>
#include <vector>

#include "moe_gemm.cuh"

using namespace l4moe;

struct Group {
    int rows, expert;
};

// The table the permutation kernel writes: heavy groups first, then light,
// each run in candidate order, empty groups left out.
static void make_table(GroupTable& tab, const std::vector<Group>& cand, int fb_routed, int fb_shared,
                       int ksplit, int E) {
    int n = 0, t = 0;
    for (int run = 0; run < 2; ++run) {
        for (const Group& g : cand) {
            if (g.rows <= 0 || (g.rows >= kHeavyRows) != (run == 0)) continue;
            const int fb = (g.expert == E ? fb_shared : fb_routed) * ksplit;
            tab.rows[n] = g.rows;
            tab.row0[n] = 0;
            tab.expert[n] = g.expert;
            tab.tile_start[n] = t;
            t += ((g.rows + kTokTile - 1) / kTokTile) * fb;
            ++n;
        }
        if (run == 0) tab.heavy_tiles = t;
    }
    int r0 = 0;  // rows are laid out in table order
    for (int i = 0; i < n; ++i) {
        tab.row0[i] = r0;
        r0 += tab.rows[i];
    }
    tab.num_groups = n;
    tab.total_tiles = t;
    tab.tile_start[n] = t;
}

template <int MODE>
static bool run_case(std::mt19937& rng, int c) {
    const int E = 1 + (int)(rng() % 40);
    const int BK = 64;  // bf16 k-block
    const int K_r = BK * (1 + (int)(rng() % 130)), K_s = BK * (1 + (int)(rng() % 130));
    const int M_r = 64 * (1 + (int)(rng() % 40)), M_s = 64 * (1 + (int)(rng() % 40));
    const int ksplit = 1 + (int)(rng() % 4);
    std::vector<Group> cand;
    const int mode = rng() % 3;
    for (int e = 0; e < E; ++e) {
        int rows = 0;
        if (rng() % 4 != 0)
            rows = mode == 0 ? 1 + (int)(rng() % 300) : mode == 1 ? 1 + (int)(rng() % 3000) : (int)(rng() % 40);
        cand.push_back({rows, e});
    }
    cand.push_back({1 + (int)(rng() % 5000), E});  // the shared expert
    const int fb_r = (M_r + pair_features<MODE>() - 1) / pair_features<MODE>();
    const int fb_s = (M_s + pair_features<MODE>() - 1) / pair_features<MODE>();
    GroupTable tab{};
    make_table(tab, cand, fb_r, fb_s, ksplit, E);
    GemmArgs a{};
    a.num_experts = E;
    a.k_routed = K_r;
    a.k_shared = K_s;
    a.m_routed = M_r;
    a.m_shared = M_s;
    a.ksplit = ksplit;
    std::set<std::tuple<int, int, int, int>> seen;
    for (int L = 0; L < tab.total_tiles; ++L) {
        const TileInfo ti = decode_tile<MODE, 64, 2>(tab, a, L);
        int g = -1;
        for (int i = 0; i < tab.num_groups; ++i)
            if (tab.expert[i] == ti.expert) g = i;
        const bool sh = ti.expert == E;
        const int rel = ti.row0 - (g >= 0 ? tab.row0[g] : 0);
        const int nkb = (sh ? K_s : K_r) / BK;
        const bool ok = g >= 0 && ti.shared == sh && rel >= 0 && rel % kTokTile == 0 && rel < tab.rows[g] &&
                        ti.n_valid == std::min(kTokTile, tab.rows[g] - rel) && ti.n_mma >= ti.n_valid &&
                        ti.n_mma % 16 == 0 && ti.n_mma <= kTokTile && ti.f0 >= 0 && ti.f0 % pair_features<MODE>() == 0 &&
                        ti.f0 < (sh ? M_s : M_r) && ti.split >= 0 && ti.split < ksplit &&
                        ti.kb0 == (int)((long long)nkb * ti.split / ksplit) &&
                        ti.kb1 == (int)((long long)nkb * (ti.split + 1) / ksplit) && ti.K == (sh ? K_s : K_r) &&
                        ti.M == (sh ? M_s : M_r);
        if (!ok || !seen.insert({ti.expert, ti.row0, ti.f0, ti.split}).second) {
            printf("BAD mode %d case %d L %d: expert %d row0 %d n_valid %d f0 %d split %d kb [%d,%d)\n", MODE, c,
                   L, ti.expert, ti.row0, ti.n_valid, ti.f0, ti.split, ti.kb0, ti.kb1);
            return false;
        }
    }
    // every (group, token tile, feature block, split) appears
    long long want = 0;
    for (int i = 0; i < tab.num_groups; ++i)
        want += (long long)((tab.rows[i] + kTokTile - 1) / kTokTile) *
                (tab.expert[i] == E ? fb_s : fb_r) * ksplit;
    if ((long long)seen.size() != want || want != tab.total_tiles) {
        printf("BAD mode %d case %d: %zu tiles decoded, %lld expected\n", MODE, c, seen.size(), want);
        return false;
    }
    return true;
}

// A small batch's table (shared expert first, then the routed experts in
// index order, every group light): the shared expert's tiles decoded without
// the table equal the table's first tiles.
template <int MODE>
static bool early_case(std::mt19937& rng, int c) {
    const int E = 1 + (int)(rng() % 256);
    const int T = 1 + (int)(rng() % 16), k = 1 + (int)(rng() % 4);
    const int ksplit = 1 + (int)(rng() % 16);
    const int K_r = 64 * (1 + (int)(rng() % 130)), K_s = 64 * (1 + (int)(rng() % 130));
    const int M_r = 64 * (1 + (int)(rng() % 160)), M_s = 64 * (1 + (int)(rng() % 160));
    std::vector<Group> cand;
    cand.push_back({T, E});
    for (int e = 0; e < E; ++e) cand.push_back({(rng() % 8 == 0) ? (int)(rng() % (T * k + 1)) : 0, e});
    const int fb_r = (M_r + pair_features<MODE>() - 1) / pair_features<MODE>();
    const int fb_s = (M_s + pair_features<MODE>() - 1) / pair_features<MODE>();
    GroupTable tab{};
    make_table(tab, cand, fb_r, fb_s, ksplit, E);
    GemmArgs a{};
    a.num_experts = E;
    a.k_routed = K_r;
    a.k_shared = K_s;
    a.m_routed = M_r;
    a.m_shared = M_s;
    a.ksplit = ksplit;
    const int early = ((T + kTokTile - 1) / kTokTile) * fb_s * ksplit;
    if (tab.heavy_tiles != 0 || tab.expert[0] != E || tab.tile_start[1] != early) {
        printf("BAD early case %d: table does not lead with the shared expert\n", c);
        return false;
    }
    for (int L = 0; L < early; ++L) {
        const TileInfo x = decode_in_group<MODE, 64, 2>(a, T, 0, E, early, L);
        const TileInfo y = decode_tile<MODE, 64, 2>(tab, a, L);
        if (x.expert != y.expert || x.row0 != y.row0 || x.n_valid != y.n_valid || x.n_mma != y.n_mma ||
            x.f0 != y.f0 || x.K != y.K || x.M != y.M || x.up_off != y.up_off || x.split != y.split ||
            x.kb0 != y.kb0 || x.kb1 != y.kb1 || x.shared != y.shared) {
            printf("BAD early case %d L %d\n", c, L);
            return false;
        }
    }
    return true;
}

int main() {
    std::mt19937 rng(2024);
    int cases = 0;
    for (int c = 0; c < 2000; ++c) {
        if (!early_case<MODE_GATEUP>(rng, c) || !early_case<MODE_DOWN>(rng, c)) return 1;
        cases += 2;
    }
    // tile_at alone: a permutation of [0, total) that keeps each run's order
    for (int total = 1; total <= 300; ++total)
        for (int heavy = 0; heavy <= total; ++heavy) {
            std::vector<int> hit(total, 0);
            int last_h = -1, last_l = heavy - 1;
            for (int L = 0; L < total; ++L) {
                const int t = tile_at(L, heavy, total);
                if (t < 0 || t >= total || hit[t]++) {
                    printf("BAD tile_at(%d, %d, %d) = %d\n", L, heavy, total, t);
                    return 1;
                }
                if (t < heavy) {
                    if (t != last_h + 1) { printf("BAD heavy order at %d/%d\n", heavy, total); return 1; }
                    last_h = t;
                } else {
                    if (t != last_l + 1) { printf("BAD light order at %d/%d\n", heavy, total); return 1; }
                    last_l = t;
                }
            }
            ++cases;
        }
    for (int c = 0; c < 3000; ++c) {
        if (!run_case<MODE_GATEUP>(rng, c) || !run_case<MODE_DOWN>(rng, c)) return 1;
        cases += 2;
    }
    printf("OK %d\n", cases);
    return 0;
}
