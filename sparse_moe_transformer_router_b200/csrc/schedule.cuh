// schedule.cuh -- the work list a grouped GEMM launch reads (written by the
// permutation kernel) and the order in which its tiles are taken.
#pragma once

namespace l4moe {

// One GEMM launch's work list: the non-empty groups (a routed expert or the
// shared expert), the rows each group owns in its activation matrix, and the
// first tile of each group in the launch's linear tile order.  Tiles of a
// group are (feature block) x (token block); group g holds
// ceil(rows/kTokTile) * feature_blocks tiles.
constexpr int kMaxGroups = 257;  // 256 routed experts + the shared expert
constexpr int kTokTile = 256;    // tokens per GEMM tile (MMA N, swap-AB)

// Groups are listed in two runs: first the "heavy" groups (at least
// kHeavyRows rows: enough tokens per weight tile that the tensor cores, not
// the weight stream, bound them), then the light ones.  The GEMM interleaves
// the two runs' tiles evenly (see tile_at), so compute-bound and
// weight-stream-bound tiles run side by side instead of in separate phases.
constexpr int kHeavyRows = 192;

struct GroupTable {
    int num_groups;
    int total_tiles;
    int heavy_tiles;  // tiles of the leading heavy run: tile_start[first light group]
    int pad0;
    int rows[kMaxGroups];
    int row0[kMaxGroups];
    int expert[kMaxGroups];       // 0..E-1 routed, E = shared
    int tile_start[kMaxGroups + 1];
};

// Launch position L (0 .. total-1) -> tile number in the table's order.  The
// heavy run's H tiles take the positions where floor((L+1) H / N) steps up,
// spread as evenly as integers allow, the light run's tiles the others; both
// runs keep their own order, so tiles that share a weight tile stay close.
__host__ __device__ __forceinline__ int tile_at(int L, int heavy, int total) {
    const long long h1 = ((long long)(L + 1) * heavy) / total;
    const long long h0 = ((long long)L * heavy) / total;
    return h1 > h0 ? (int)(h1 - 1) : heavy + (L - (int)h1);
}

}  // namespace l4moe
