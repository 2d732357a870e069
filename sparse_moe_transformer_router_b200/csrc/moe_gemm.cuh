// moe_gemm.cuh -- persistent grouped GEMM on the 5th-generation tensor cores
// (tcgen05 on CTA pairs, TMEM accumulators, TMA-fed shared-memory pipeline)
// for the two contractions of the layer:
//
//   gate/up  : a = g * (x . W_gate_up)  then h = silu(a[:F]) * a[F:]
//              (SwiGLU), for the shared expert (g = 1) and every routed
//              expert (x rows in expert order, g = the token's sigmoid gate,
//              applied to the fp32 accumulator: the gate scales the input
//              and the contraction is linear in it) in one launch
//   down     : y = h . W_down for the shared expert (all tokens) and every
//              routed expert in one launch; each tile stores its fp32 result
//              un-permuted to the token's row of a partial buffer, and a
//              finish kernel writes out = rn(y_shared + y_routed), one rounding
//
// llm-architectures-explained "Llama 4 Maverick", field table rows
// ffns.moe.gated / d_expert / d_shared: every expert and the shared expert is
// a gated MLP of width 8192; superteams.ai "Llama 4" glossary, routing
// sketch: the layer output is the shared expert's output plus the routed
// expert's.
//
// Orientation ("swap-AB"): the weight is the MMA A operand (output features
// as M, read MN-major straight from the row-major [K, N] weight) and the
// activations are the B operand (tokens as N, up to 256, K-major rows).  A
// group's token count is only padded to a multiple of 16, so ragged experts
// (and decode, T <= 128) waste little tensor work.
//
// CTA pairs (cluster of 2, cta_group::2): one MMA computes M = 256 rows x N
// tokens; each CTA loads its own 128 A rows and its own half of the N tokens
// into its shared memory and holds its 128 rows x N columns of the fp32
// accumulator in its TMEM.  Per SM that halves the token operand each tile
// streams through L2 compared with a single-CTA 128-row tile.
//   down   : pair tile = 256 output features (128 per CTA).
//   gate/up: pair tile = 128 features; each CTA's 128 A rows are the gate
//            rows (64 features) followed by the up rows of the same 64
//            features, so TMEM lane r holds gate and lane r + 64 holds up;
//            the epilogue pairs them through a small shared-memory exchange.
// Accumulators are double-buffered (2 x 256 TMEM columns) so the epilogue of
// one tile overlaps the MMAs of the next.
//
// E4M3 weights (FP8W): TMA brings the raw 8-bit A tile (64 K rows x 2 slabs
// of 64 features) into a raw ring; eight converter warps widen it exactly to
// f16, write the swizzled MN-major operand layout, fence to the async proxy
// and report to the leader; the MMA (kind::f16, both operands f16: these
// layers keep their token operand and hidden rows in f16) waits for the
// token tile and for both CTAs' converted weights, and the epilogue
// multiplies each accumulator row by its weight column's fp32 scale.
//
// FP8 activation mode (WQ = kWqAct8): the weights are E4M3 codes and so
// are the token rows (x quantised per row while it is permuted, the hidden
// rows quantised per row by their own kernel), and the MMA takes both raw:
// kind::f8f6f4, 128 K per stage (one 128-byte token row), the weight tile as
// two 64-feature slabs in the 64-byte swizzle (a slab row is 64 features of
// one K row), no converter warps.  The epilogue multiplies each accumulator
// row by its weight column's scale and each column by its token row's scale
// (gate/up: the sigmoid gate times the x row's scale, through the same
// column-scale path as the gate; down: the hidden row's scale).
//
// Tiles: a group's tiles are (feature block) x (token tile) x (k range), the
// token tiles of one feature block adjacent so that they share the weight
// tile through L2, in bands whose token rows stay in L2 while the band
// sweeps the feature blocks; compute-bound and weight-bound groups are
// interleaved (tile_at); CTA pairs take tiles in stripes.  The token operand
// arrives as one 128-row box per k-block for tiles of more than 64 tokens
// per CTA (measured: a box's issue cost dominated with 64-row boxes), else
// as 32-row boxes.
//
// Roles (320 threads per CTA; 448 with widened coded weights): warp 0 lane 0
// issues TMA loads into a STAGES-deep ring (both CTAs; completion counted on
// the leader's barrier); warp 1 allocates TMEM (both CTAs) and, in the
// leader CTA only, lane 0 issues the MMAs and commits to both CTAs'
// barriers; warps 2..9 are the epilogue (warp w reads TMEM lanes
// 32*(w%4) .. +31, the two warps of a lane quarter alternate 32-column
// chunks; with widened coded weights warps 2..5 alone, one per quarter,
// then the converter warps) and release the accumulator to the leader.  Every mbarrier wait is bounded: on a timeout a
// role records a bit in the error word and returns; the leader drains the
// copies and MMAs in flight before the pair synchronises and frees TMEM.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "schedule.cuh"

namespace l4moe {

// MODE_FUSED: one launch takes the gate/up tiles and then the down tiles of
// a small batch (see TileCursor and the down tiles' wait in the producer).
enum GemmMode : int { MODE_GATEUP = 0, MODE_DOWN = 1, MODE_FUSED = 2 };

// The MMA operand type's tiling: K per stage (one 128-byte token row), K per
// MMA, the instruction's format code, and the MN-major weight tile's slabs
// (A_BOX_FEATS features per slab row, one TMA box per slab) and swizzle.
template <typename ET>
struct ElemCfg;
template <>
struct ElemCfg<__nv_bfloat16> {
    static constexpr int BYTES = 2;
    static constexpr int BK = 64;     // K elements per stage (one 128-byte row)
    static constexpr int MMA_K = 16;  // K per tcgen05.mma (kind::f16)
    static constexpr uint32_t FMT = 1;
    static constexpr int A_BOX_FEATS = 64;    // one 128-byte slab row
    static constexpr uint32_t A_LAYOUT = 2;   // MN-major weights: 128B swizzle, 16B unit
    static constexpr uint32_t A_SBO = 1024;   // 8 K rows per atom
};
template <>
struct ElemCfg<float> {
    static constexpr int BYTES = 4;
    static constexpr int BK = 32;
    static constexpr int MMA_K = 8;   // kind::tf32
    static constexpr uint32_t FMT = 2;
    static constexpr int A_BOX_FEATS = 32;
    static constexpr uint32_t A_LAYOUT = 1;   // MN-major 32-bit: 128B swizzle, 32B unit
    static constexpr uint32_t A_SBO = 512;    // 4 K rows per atom
};
// E4M3 codes on both sides (the FP8 activation mode)
struct E4M3Op {};
template <>
struct ElemCfg<E4M3Op> {
    static constexpr int BYTES = 1;
    static constexpr int BK = 128;
    static constexpr int MMA_K = 32;  // kind::f8f6f4
    static constexpr uint32_t FMT = 0;        // E4M3
    static constexpr int A_BOX_FEATS = 64;    // [gate 64 | up 64] stays two slabs
    static constexpr uint32_t A_LAYOUT = 4;   // MN-major: 64B swizzle, slab rows of 64 bytes
    static constexpr uint32_t A_SBO = 512;    // 8 K rows per atom
};

struct GemmArgs {
    const GroupTable* table;
    const CUtensorMap* a_maps;  // weights, [E + 1]: routed experts then the shared expert
    int num_experts;            // E (expert index E = shared)
    int k_routed, k_shared;     // reduction length per class (gate/up: d, d; down: F, Fs)
    int m_routed, m_shared;     // output features per class (F / Fs, or d)
    int up_routed, up_shared;   // gate/up: column offset of the "up" half (F / Fs)
    void* out_routed;
    long long ld_routed;
    void* out_shared;
    long long ld_shared;
    const int32_t* rowmap_routed;  // down: output row (token) of a slot (perm), else null
    const int32_t* rowmap_shared;  // gate/up: slot of a token (inv); down: perm
    const float* colscale_routed;  // gate/up: sigmoid gate of each slot (times its row's scale), else null
    const float* colscale_shared;  // gate/up, 8-bit weights: power-of-two scale of each token's f16 row, else null
    const float* const* wscale;    // E4M3 weights: per-column scale vector of each of the
                                   // E + 1 weight matrices of this launch, else null
    // fp32 partial output (always for down; for gate/up when split): each
    // tile covers k-block range s of ksplit (split-K when tiles are few, e.g.
    // decode) and stores its fp32 result; a finish kernel sums the partials
    int ksplit;                    // 1 = no split
    int partial_out;               // store fp32 partials instead of the epilogue's output
    float* part_routed;            // [ksplit][rows][ld_part_routed] fp32, or null
    long long ld_part_routed;
    float* part_shared;            // gate/up only: shared expert partials
    long long ld_part_shared;
    long long part_stride_routed;  // elements between splits
    long long part_stride_shared;
    unsigned* err;
    // early start (gate/up after the small-batch routing, shared operand x):
    // the leading early_tiles positions are the shared expert's tiles over
    // early_rows tokens, run before the routing has finished; 0 = none
    int early_tiles;
    int early_rows;
    // fused launches: [0] shared, [1] routed gate/up epilogue warps done
    // (each warp of both CTAs counts once per tile; zero when the launch
    // starts, reset by the down finish kernel)
    unsigned* done;
};

// Output features covered by one pair tile.
template <int MODE>
__host__ __device__ constexpr int pair_features() { return MODE == MODE_GATEUP ? 128 : 256; }

// Weight storage of a GEMM: the layer's own type, or 8-bit or 4-bit codes
// widened in shared memory (E4M3 floats, int8 or int4 integers, per-column
// scales).
// kWqAct8: E4M3 weights read raw by an MMA on E4M3 token rows (the FP8
// activation mode).
enum : int { kWqNone = 0, kWqE4M3 = 1, kWqInt8 = 2, kWqInt4 = 3, kWqAct8 = 4 };

// The MMA operand type of a GEMM: the layer's type, or E4M3 codes.
template <typename ET, int WQ>
struct OperandOf {
    using type = ET;
};
template <typename ET>
struct OperandOf<ET, kWqAct8> {
    using type = E4M3Op;
};

// SMALLN: every tile of the launch has at most 2 * B_SMALL_ROWS token rows
// (small batches: decode).  The token operand then needs one 32-row box per
// CTA and stage, so a stage shrinks to the weight tile plus 4 KB and the ring
// holds more stages: these launches stream weights, and the bytes in flight
// per SM set how much of the HBM bandwidth they reach.
template <int MODE, typename ET, int WQ, bool SMALLN = false>
struct GemmCfg {
    static constexpr bool ACT8 = WQ == kWqAct8;               // E4M3 x E4M3, raw operands
    static constexpr bool FP8W = WQ != kWqNone && !ACT8;      // coded weights, converter warps
    using C = ElemCfg<typename OperandOf<ET, WQ>::type>;
    static constexpr int A_BYTES = 128 * 128;                // 128 A rows x 128 B of K
    static constexpr int A_BOX_FEATS = C::A_BOX_FEATS;       // features per A box (one slab)
    static constexpr int A_BOXES = 128 / A_BOX_FEATS;        // boxes per CTA A tile
    static constexpr int A_ROW_BYTES = A_BOX_FEATS * C::BYTES;  // bytes of one K row of a slab
    static constexpr int A_BOX_BYTES = C::BK * A_ROW_BYTES;  // BK rows of a slab
    static constexpr int B_BOX_ROWS = 128;                   // token rows per full-tile box
    static constexpr int B_SMALL_ROWS = 32;                  // token rows per small-tile box
    static constexpr int B_BYTES = (SMALLN ? B_SMALL_ROWS : kTokTile / 2) * 128;  // this CTA's token rows
    // raw coded weights: 2 slabs x 64 K rows x 64 features, one byte per code
    // (half a byte for int4: two codes per byte along the features)
    static constexpr int RAW_SLAB_BYTES = WQ == kWqInt4 ? 64 * 32 : 64 * 64;
    static constexpr int RAW_BYTES = FP8W ? 2 * RAW_SLAB_BYTES : 0;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + RAW_BYTES;
    static constexpr int STAGES = SMALLN ? (FP8W ? 7 : 10) : (FP8W ? 5 : 6);
    static constexpr int ACC_BUFS = 2;
    static constexpr int TMEM_COLS = 512;
    // epilogue warps: one per TMEM lane quarter, or two (each taking every
    // other 32-column chunk) where a tile's mainloop is short enough that
    // one warp per quarter cannot keep up (the E4M3 x E4M3 tiles: half the
    // k-blocks of a bf16 tile for the same epilogue work)
    static constexpr int EPI_WARPS = FP8W ? 4 : 8;
    static constexpr int EPI_HALVES = EPI_WARPS / 4;
    static constexpr int CONV_WARPS = FP8W ? 8 : 0;         // widening warps (after the epilogue's)
    static constexpr int CONV_WARP0 = 2 + EPI_WARPS;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS + 32 * CONV_WARPS;
    static constexpr int XLD = 17;                           // exchange row stride (floats)
    static constexpr int XCH_FLOATS = 2 * 2 * 32 * XLD;      // one half's exchange buffers
    static constexpr int XCH_BYTES = (MODE != MODE_DOWN) ? EPI_HALVES * XCH_FLOATS * 4 : 0;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * ACC_BUFS + 1 + (FP8W ? 2 * STAGES : 0);
    static constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES +
                                         XCH_BYTES + NUM_BARS * 8 + 16 + sizeof(GroupTable);
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
};

struct TileInfo {
    int mode;  // 0: a gate/up tile, 1: a down tile
    int expert, row0, n_valid, n_mma, f0, K, M, up_off;
    int split, kb0, kb1;  // k-block range [kb0, kb1) of this tile's split
    bool shared;
};

// Activation bytes a band of token tiles may keep in L2 (each of the two
// dies caches what its SMs read, so this stays well under half of L2).
constexpr long long kBandBytes = 24ll << 20;

// Tile `local` of a group: `rows` activation rows from `row0`, weights of
// `expert`, `group_tiles` tiles in all.
template <int MODE, int ElemCfgBK, int ElemBytes>
__host__ __device__ __forceinline__ TileInfo decode_in_group(const GemmArgs& a, int rows, int row0, int expert,
                                                             int group_tiles, int local) {
    const int ntb = (rows + kTokTile - 1) / kTokTile;
    TileInfo ti;
    ti.mode = MODE == MODE_DOWN ? 1 : 0;
    ti.expert = expert;
    ti.shared = (ti.expert == a.num_experts);
    ti.K = ti.shared ? a.k_shared : a.k_routed;
    // Token tiles go in bands of `band` tiles whose activation rows (the B
    // operand, about kBandBytes) stay in L2 while the band sweeps every
    // feature block; inside a band the token tile varies fastest, so the
    // tiles that share a weight tile run side by side.
    const int band = max(1, (int)(kBandBytes / ((long long)kTokTile * ti.K * ElemBytes)));
    const int fbk = group_tiles / ntb;  // feature blocks x splits
    const int b = local / (band * fbk);
    const int nb = min(band, ntb - b * band);  // token tiles in this band (the last may be short)
    const int rem = local - b * band * fbk;
    const int tb = b * band + rem % nb;
    const int rest = rem / nb;
    // split-K units go split-major: the units that run side by side cover
    // different feature blocks (column bands of the weight) instead of
    // different K rows of one band, spreading their weight stream over the
    // memory channels
    const int nfb = fbk / a.ksplit;  // feature blocks
    const int fb = rest % nfb;
    const int split = rest / nfb;
    ti.split = split;
    ti.row0 = row0 + tb * kTokTile;
    ti.n_valid = min(kTokTile, rows - tb * kTokTile);
    ti.n_mma = (ti.n_valid + 15) & ~15;
    ti.f0 = fb * pair_features<MODE>();
    ti.M = ti.shared ? a.m_shared : a.m_routed;
    ti.up_off = ti.shared ? a.up_shared : a.up_routed;
    const int nkb = (ti.K + ElemCfgBK - 1) / ElemCfgBK;  // a ragged last block reads zeros
    ti.kb0 = (int)(((long long)nkb * split) / a.ksplit);
    ti.kb1 = (int)(((long long)nkb * (split + 1)) / a.ksplit);
    return ti;
}

// Launch position `pos` -> its tile, through the work list.
template <int MODE, int ElemCfgBK, int ElemBytes>
__host__ __device__ __forceinline__ TileInfo decode_tile(const GroupTable& tab, const GemmArgs& a, int pos) {
    const int L = tile_at(pos, tab.heavy_tiles, tab.total_tiles);
    int lo = 0, hi = tab.num_groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab.tile_start[mid] <= L) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    return decode_in_group<MODE, ElemCfgBK, ElemBytes>(a, tab.rows[g], tab.row0[g], tab.expert[g],
                                                       tab.tile_start[g + 1] - tab.tile_start[g],
                                                       L - tab.tile_start[g]);
}

// The tiles of one launch as a role walks them.  Normally every tile comes
// from the work list, copied to shared memory once the kernel that writes it
// has finished (the wait at kernel entry).  With early_tiles > 0 the launch
// starts before that kernel has finished: its first early_tiles positions
// are the shared expert's tiles (rows 0 .. early_rows of the shared operand,
// which that kernel does not write), decoded without the work list; the
// first position past them waits for the preceding kernel (griddepcontrol)
// and from there on decodes through the work list in global memory.  A
// fused launch (always early) continues past the gate/up work list's tiles
// with the down work list's.
template <int MODE, int ElemCfgBK, int ElemBytes>
struct TileCursor {
    static constexpr int GU = MODE == MODE_FUSED ? MODE_GATEUP : MODE;  // mode of the first work list
    const GroupTable* tab;  // shared-memory copy (not early)
    int total;              // tiles of the launch
    int n_first;            // tiles of the first (gate/up, or the only) work list
    bool waited;

    __device__ __forceinline__ TileCursor(const GroupTable* smem_tab, const GemmArgs& a)
        : tab(smem_tab),
          total(a.early_tiles > 0 ? 0x7FFFFFFF : smem_tab->total_tiles),
          n_first(a.early_tiles > 0 ? 0x7FFFFFFF : smem_tab->total_tiles),
          waited(a.early_tiles == 0) {}

    __device__ __forceinline__ TileInfo tile(const GemmArgs& a, const GemmArgs& dn, int L) const {
        if (L < a.early_tiles)
            return decode_in_group<GU, ElemCfgBK, ElemBytes>(a, a.early_rows, 0, a.num_experts, a.early_tiles, L);
        if (L < n_first) return decode_tile<GU, ElemCfgBK, ElemBytes>(a.early_tiles > 0 ? *a.table : *tab, a, L);
        return decode_tile<MODE_DOWN, ElemCfgBK, ElemBytes>(*dn.table, dn, L - n_first);
    }

    // Tile at position L, or false past the last one.
    __device__ __forceinline__ bool at(const GemmArgs& a, const GemmArgs& dn, int L, TileInfo& ti) {
        if (!waited && L >= a.early_tiles) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited = true;
            n_first = a.table->total_tiles;
            total = n_first + (MODE == MODE_FUSED ? dn.table->total_tiles : 0);
        }
        if (L >= total) return false;
        ti = tile(a, dn, L);
        return true;
    }
    // The weight descriptor of the tile at L when it can be known now (else null).
    __device__ __forceinline__ const CUtensorMap* map_if_known(const GemmArgs& a, const GemmArgs& dn, int L) const {
        if (L < a.early_tiles) return a.a_maps + a.num_experts;
        if (!waited || L >= total) return nullptr;
        const TileInfo t = tile(a, dn, L);
        return (t.mode ? dn.a_maps : a.a_maps) + t.expert;
    }
};

// Bounded wait until *count >= target (acquire), for a fused launch's down
// tiles; on a timeout the producer's bit is set in the error word.
__device__ __forceinline__ uint32_t ld_acquire_gpu(const unsigned* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ bool wait_count(const unsigned* count, unsigned target, unsigned* err) {
    if (ld_acquire_gpu(count) >= target) return true;
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_gpu(count) < target) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, DEV_ERR_TIMEOUT_PRODUCER);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// 8 E4M3 codes (little-endian in a uint2) -> 8 f16 values, exactly (every
// E4M3 value, subnormals included, is an f16 value), with the hardware
// conversion (two codes per instruction, element order kept).  The
// per-column scale is applied to the fp32 accumulator in the epilogue.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    uint32_t r;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
        : "=r"(r)
        : "r"(two_codes));
    return r;
}

__device__ __forceinline__ uint4 e4m3x8_to_f16(uint2 raw) {
    return make_uint4(e4m3x2_to_f16x2(raw.x & 0xFFFFu), e4m3x2_to_f16x2(raw.x >> 16),
                      e4m3x2_to_f16x2(raw.y & 0xFFFFu), e4m3x2_to_f16x2(raw.y >> 16));
}

// 8 int8 codes (little-endian in a uint2) -> 8 f16 values, exactly.  With
// the code biased to u = q + 128 in [0, 255] (flipping bit 7), the f16 whose
// high byte is 0x64 and low byte is u has exponent 10 and value 1024 + u (u
// fills the low mantissa bits); subtracting 1152 = 1024 + 128 leaves q, and
// both values and the difference are integers below 2^11, so every step is
// exact.  Two bytes per byte permutation and per f16x2 subtraction.
__device__ __forceinline__ uint32_t i8x2_to_f16x2(uint32_t biased4, uint32_t sel) {
    uint32_t h, r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(h) : "r"(biased4), "r"(0x64646464u), "r"(sel));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64806480u));
    return r;
}

__device__ __forceinline__ uint4 int8x8_to_f16(uint2 raw) {
    const uint32_t lo = raw.x ^ 0x80808080u, hi = raw.y ^ 0x80808080u;
    // byte selectors: (code byte, 0x64, code byte, 0x64) from the low / high pair
    return make_uint4(i8x2_to_f16x2(lo, 0x4140u), i8x2_to_f16x2(lo, 0x4342u),
                      i8x2_to_f16x2(hi, 0x4140u), i8x2_to_f16x2(hi, 0x4342u));
}

// 8 int4 codes (two's complement nibbles, the lower-numbered code in the low
// nibble of each byte, bytes little-endian in a uint32) -> 8 f16 values,
// exactly.  As for int8: flipping each nibble's sign bit gives u = q + 8 in
// [0, 15]; the f16 with high byte 0x64 and low bits u has the value 1024 + u,
// and subtracting 1032 = 1024 + 8 leaves q (every value an integer below
// 2^11, so every step is exact).  Byte i of the biased word holds the pair
// (code 2i, code 2i+1): its low nibble goes to the low f16 of the pair, its
// high nibble to the high f16.
__device__ __forceinline__ uint32_t i4pair_to_f16x2(uint32_t biased, int byte) {
    const uint32_t t = biased >> (8 * byte);
    const uint32_t h = (t & 0x0Fu) | ((t & 0xF0u) << 12) | 0x64006400u;
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64086408u));
    return r;
}

__device__ __forceinline__ uint4 int4x8_to_f16(uint32_t raw) {
    const uint32_t b = raw ^ 0x88888888u;
    return make_uint4(i4pair_to_f16x2(b, 0), i4pair_to_f16x2(b, 1), i4pair_to_f16x2(b, 2),
                      i4pair_to_f16x2(b, 3));
}


// The contractions' activation (token operand and hidden) type: the layer's
// own, or f16 for E4M3 weights (kind::f16 takes both operands in one type).
template <typename ET, bool FP8W>
struct GemmAct {
    using type = ET;
};
template <>
struct GemmAct<__nv_bfloat16, true> {
    using type = __half;
};

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
__device__ __forceinline__ void store_elem(__half* p, float v) { *p = __float2half_rn(v); }

// Token-operand (B) descriptors of the routed and the shared rows, with
// 128-row boxes for tiles of more than 64 tokens per CTA and 32-row boxes
// for the others.  A box always lands whole (zero-filled past the matrix), so
// the box size sets the bytes a small tile moves; one big box instead of
// several small ones keeps the TMA unit's per-box cost off the full tiles.
struct BMaps {
    CUtensorMap routed, shared, routed_small, shared_small;
};

template <int MODE, typename ET, int WQ, bool SMALLN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GemmCfg<MODE, ET, WQ, SMALLN>::THREADS, 1)
    moe_gemm_kernel(const __grid_constant__ BMaps bm, const __grid_constant__ GemmArgs args,
                    const __grid_constant__ BMaps bm_dn, const __grid_constant__ GemmArgs args_dn) {
    // bm / args: the launch's GEMM, or a fused launch's gate/up; bm_dn /
    // args_dn: a fused launch's down (unused otherwise)
    // early start: the work list is read after the first wait (TileCursor)
    if (args.early_tiles > 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    else pdl_enter();
    using Cfg = GemmCfg<MODE, ET, WQ, SMALLN>;
    constexpr bool FP8W = Cfg::FP8W;      // coded (8- or 4-bit) weights with converter warps
    constexpr bool ACT8 = Cfg::ACT8;      // E4M3 weights and token rows, read raw
    constexpr bool WSC = WQ != kWqNone;   // per-column weight scales in the epilogue
    using C = typename Cfg::C;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float* xch = reinterpret_cast<float*>(smem + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES +
                                                 Cfg::XCH_BYTES);
    uint32_t* misc = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);  // [0] TMEM base, [1] abort
    GroupTable* tab = reinterpret_cast<GroupTable*>(misc + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer
    const bool leader = rank == 0;
    const uint32_t stage0 = smem_u32(smem);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (Cfg::STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * Cfg::STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * Cfg::STAGES + Cfg::ACC_BUFS + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * Cfg::STAGES + 2 * Cfg::ACC_BUFS);
    // E4M3 weights: raw tile landed (local) / both CTAs' converted tile ready (leader)
    auto rawfull_bar = [&](int s) { return bar0 + 8u * (2 * Cfg::STAGES + 2 * Cfg::ACC_BUFS + 1 + s); };
    auto conv_bar = [&](int s) {
        return bar0 + 8u * (3 * Cfg::STAGES + 2 * Cfg::ACC_BUFS + 1 + s);
    };

    if (args.early_tiles == 0) {  // work list -> shared memory
        const int* src = reinterpret_cast<const int*>(args.table);
        int* dst = reinterpret_cast<int*>(tab);
        for (int i = threadIdx.x; i < (int)(sizeof(GroupTable) / 4); i += blockDim.x) dst[i] = src[i];
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(full_bar(s), 1);   // leader: one expect_tx arrival for both CTAs' bytes
            mbar_init(empty_bar(s), 1);  // one multicast commit per use
        }
        for (int b = 0; b < Cfg::ACC_BUFS; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 2 * Cfg::EPI_WARPS);  // leader: the epilogue warps of each CTA
        }
        mbar_init(drain_bar, 1);
        if constexpr (FP8W) {
            for (int s = 0; s < Cfg::STAGES; ++s) {
                mbar_init(rawfull_bar(s), 1);
                mbar_init(conv_bar(s), 2 * Cfg::CONV_WARPS);  // leader: converter warps of both CTAs
            }
        }
        misc[1] = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&bm.routed);
        tma_prefetch_desc(&bm.shared);
        tma_prefetch_desc(&bm.routed_small);
        tma_prefetch_desc(&bm.shared_small);
        if constexpr (MODE == MODE_FUSED) {
            tma_prefetch_desc(&bm_dn.routed);
            tma_prefetch_desc(&bm_dn.shared);
            tma_prefetch_desc(&bm_dn.routed_small);
            tma_prefetch_desc(&bm_dn.shared_small);
        }
    }
    cluster_sync();  // barriers of both CTAs initialised before any remote use
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(misc), Cfg::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    using Cursor = TileCursor<MODE, C::BK, C::BYTES>;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t used = 0, last_par = 0;  // per stage: issued at least once / its parity
            bool aborted = false;
            uint32_t dep_ready = 0;  // fused: bit c set once class c's hidden rows are complete
            Cursor cur(tab, args);
            TileInfo ti;
            for (int L = pair; !aborted && cur.at(args, args_dn, L, ti); L += npairs) {
                const bool dn_tile = MODE == MODE_FUSED && ti.mode == 1;
                const GemmArgs& A = dn_tile ? args_dn : args;
                const BMaps& BM = dn_tile ? bm_dn : bm;
                const bool gu = MODE == MODE_GATEUP || (MODE == MODE_FUSED && ti.mode == 0);
                const CUtensorMap* amap = A.a_maps + ti.expert;
                // the next tile's weight descriptor, fetched while this tile streams
                // (split-K units and small groups change expert every few k-blocks)
                const CUtensorMap* next_map = cur.map_if_known(args, args_dn, L + npairs);
                if (next_map) tma_prefetch_desc(next_map);
                if constexpr (MODE == MODE_FUSED) {
                    // a down tile reads hidden rows the gate/up tiles of its class
                    // (shared or routed) write, on any CTA: wait until all of them
                    // are counted, then order this CTA's tensor-copy reads after
                    if (dn_tile) {
                        const int cls = ti.shared ? 0 : 1;
                        if (!(dep_ready >> cls & 1u)) {
                            const int tiles = cls == 0 ? args.early_tiles : cur.n_first - args.early_tiles;
                            if (!wait_count(args.done + cls, (unsigned)tiles * 2u * Cfg::EPI_WARPS, args.err)) {
                                aborted = true;
                                break;
                            }
                            asm volatile("fence.proxy.async.global;" ::: "memory");
                            dep_ready |= 1u << cls;
                        }
                    }
                }
                const int half = ti.n_mma >> 1;  // tokens per CTA
                const bool big = half > 2 * Cfg::B_SMALL_ROWS;
                const void* bmap = ti.shared ? (big ? (const void*)&BM.shared : (const void*)&BM.shared_small)
                                             : (big ? (const void*)&BM.routed : (const void*)&BM.routed_small);
                const int brows = big ? Cfg::B_BOX_ROWS : Cfg::B_SMALL_ROWS;
                const int nbb = (half + brows - 1) / brows;
                if constexpr (SMALLN) {
                    // the host launches this configuration only for tiles of at
                    // most 2 * B_SMALL_ROWS rows; anything larger would overrun the
                    // stage: report it (bad argument) and stop issuing
                    if (nbb * brows > Cfg::B_SMALL_ROWS) {
                        atomicOr(args.err, DEV_ERR_BAD_INDEX);
                        aborted = true;
                        break;
                    }
                }
                const uint32_t tx_cta =
                    (FP8W ? 0u : (uint32_t)Cfg::A_BYTES) + (uint32_t)(nbb * brows * 128);
                const int brow = ti.row0 + (int)rank * half;
                // this CTA's A columns: gate/up -> [gate 64 | up 64] of features
                // f0 + 64*rank; down -> 128 features f0 + 128*rank
                const int acol0 = gu ? ti.f0 + 64 * (int)rank : ti.f0 + 128 * (int)rank;
                for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, args.err, DEV_ERR_TIMEOUT_PRODUCER)) {
                        aborted = true;
                        break;
                    }
                    const uint32_t fb_local = full_bar(stage);
                    const uint32_t fb_leader = mapa_shared(fb_local, 0);
                    if (leader) mbar_arrive_expect_tx(fb_local, 2 * tx_cta);
                    const uint32_t sb = stage0 + (uint32_t)stage * Cfg::STAGE_BYTES;
                    const int k = kb * C::BK;
                    if constexpr (FP8W) {
                        // raw coded weights: two 64-feature slabs, signalled locally
                        // (int4: the tensor map counts bytes, two features each)
                        const uint32_t rb = sb + Cfg::A_BYTES + Cfg::B_BYTES;
                        mbar_arrive_expect_tx(rawfull_bar(stage), Cfg::RAW_BYTES);
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int col = gu ? (j == 0 ? acol0 : ti.up_off + acol0) : acol0 + 64 * j;
                            tma_load_2d(rb + j * Cfg::RAW_SLAB_BYTES, amap, rawfull_bar(stage),
                                        WQ == kWqInt4 ? col / 2 : col, k);
                        }
                    } else {
#pragma unroll
                        for (int bx = 0; bx < Cfg::A_BOXES; ++bx) {
                            int col;
                            if (gu) {
                                const int j = bx * Cfg::A_BOX_FEATS;  // 0..127 within [gate 64 | up 64]
                                col = (j < 64 ? 0 : ti.up_off - 64) + acol0 + j;
                            } else {
                                col = acol0 + bx * Cfg::A_BOX_FEATS;
                            }
                            tma_load_2d_pair(sb + bx * Cfg::A_BOX_BYTES, amap, fb_leader, col, k);
                        }
                    }
                    const uint32_t bb = sb + Cfg::A_BYTES;
                    for (int j = 0; j < nbb; ++j)
                        tma_load_2d_pair(bb + (uint32_t)(j * brows * 128), bmap, fb_leader, k,
                                         brow + j * brows);
                    used |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if constexpr (FP8W) {  // raw weight copies are counted on this CTA's barriers
                for (int s = 0; s < Cfg::STAGES; ++s)
                    if (used & (1u << s))
                        mbar_wait(rawfull_bar(s), (last_par >> s) & 1u, args.err, DEV_ERR_TIMEOUT_PRODUCER);
            }
            if (leader) {
                // the leader's full barriers count both CTAs' bytes: wait for
                // every issued copy before the pair may exit
                for (int s = 0; s < Cfg::STAGES; ++s)
                    if (used & (1u << s))
                        mbar_wait(full_bar(s), (last_par >> s) & 1u, args.err, DEV_ERR_TIMEOUT_PRODUCER);
            } else if (aborted) {
                __nanosleep(100000);  // let this CTA's own copies land before exit
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------------ MMA issuer (leader)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            Cursor cur(tab, args);
            TileInfo ti;
            for (int L = pair; cur.at(args, args_dn, L, ti); L += npairs) {
                if (!mbar_wait_cluster(tempty_bar(acc), acc_phase ^ 1u, args.err, DEV_ERR_TIMEOUT_MMA))
                    break;
                tc_fence_after();
                // 8-bit weight layers: both operands f16 (format 0), else the operand type
                const uint32_t idesc = make_idesc(FP8W ? 0u : C::FMT, 1u, 0u, (uint32_t)ti.n_mma, 256u);
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                bool ok = true;
                for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, args.err, DEV_ERR_TIMEOUT_MMA)) {
                        ok = false;
                        break;
                    }
                    if constexpr (FP8W) {
                        if (!mbar_wait(conv_bar(stage), phase, args.err, DEV_ERR_TIMEOUT_MMA)) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint32_t sb = stage0 + (uint32_t)stage * Cfg::STAGE_BYTES;
                    const uint32_t bb = sb + Cfg::A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / C::MMA_K; ++kk) {
                        const uint64_t bdesc = smem_desc(bb + kk * 32, 16, 1024, 2);
                        const uint64_t adesc = smem_desc(sb + kk * C::MMA_K * Cfg::A_ROW_BYTES,
                                                         Cfg::A_BOX_BYTES, C::A_SBO, C::A_LAYOUT);
                        const uint32_t accum = (kb != ti.kb0 || kk != 0) ? 1u : 0u;
                        if constexpr (ACT8)
                            mma_f8_pair(d_tmem, adesc, bdesc, idesc, accum);
                        else if constexpr (FP8W || C::FMT == 1)
                            mma_bf16_pair(d_tmem, adesc, bdesc, idesc, accum);
                        else
                            mma_tf32_pair(d_tmem, adesc, bdesc, idesc, accum);
                    }
                    mma_commit_pair_mc(empty_bar(stage), 0x3);  // frees the stage in both CTAs
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair_mc(tfull_bar(acc), 0x3);  // accumulator ready in both CTAs
                if (++acc == Cfg::ACC_BUFS) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every issued MMA must finish before the pair releases TMEM
            mma_commit_pair(drain_bar);
            mbar_wait(drain_bar, 0, args.err, DEV_ERR_TIMEOUT_MMA);
        }
    } else if (FP8W && warp >= Cfg::CONV_WARP0) {
        // --------------------------------------- weight-code converters (E4M3, int8, int4)
        constexpr int NCT = 32 * (Cfg::CONV_WARPS > 0 ? Cfg::CONV_WARPS : 8);  // converter threads
        static_assert(NCT == 256, "each converter thread owns 4 units: slab i / 2");
        const int ct = threadIdx.x - 32 * Cfg::CONV_WARP0;  // 0 .. NCT-1
        const int c8 = ct & 7;                      // 8-feature chunk of each slab this thread owns
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        Cursor cur(tab, args);
        TileInfo ti;
        for (int L = pair; ok && cur.at(args, args_dn, L, ti); L += npairs) {
            for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                const bool got = mbar_wait(rawfull_bar(stage), phase, args.err, DEV_ERR_TIMEOUT_PRODUCER);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const uint8_t* sbp = smem + (size_t)stage * Cfg::STAGE_BYTES;
                const uint8_t* raw = sbp + Cfg::A_BYTES + Cfg::B_BYTES;
                uint8_t* a = const_cast<uint8_t*>(sbp);
#pragma unroll
                for (int i = 0; i < 1024 / NCT; ++i) {
                    // unit u = ct + NCT i (of 2 slabs x 64 K rows x 8 chunks):
                    // slab u / 512, K row (u / 8) % 64, chunk c8
                    const int j = (i * NCT) >> 9, kr = ((ct >> 3) + (NCT / 8) * i) & 63;
                    uint4 h8;
                    if constexpr (WQ == kWqInt4) {
                        h8 = int4x8_to_f16(*reinterpret_cast<const uint32_t*>(raw + j * Cfg::RAW_SLAB_BYTES +
                                                                              kr * 32 + c8 * 4));
                    } else {
                        const uint2 q8 = *reinterpret_cast<const uint2*>(raw + j * Cfg::RAW_SLAB_BYTES + kr * 64 +
                                                                         c8 * 8);
                        if constexpr (WQ == kWqInt8) h8 = int8x8_to_f16(q8);
                        else h8 = e4m3x8_to_f16(q8);
                    }
                    *reinterpret_cast<uint4*>(a + j * 8192 + kr * 128 + ((c8 ^ (kr & 7)) << 4)) = h8;
                }
                fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(mapa_shared(conv_bar(stage), 0));
                if (++stage == Cfg::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter of this warp
        const int half = (warp - 2) >> 2;  // which 32-column chunks: half, half + halves, ...
        constexpr int CSTEP = 32 * Cfg::EPI_HALVES;
        float* xch_h = xch + half * Cfg::XCH_FLOATS;  // this half's exchange buffers
        const uint32_t bar_id = 1u + (uint32_t)half;  // this half's named barrier
        int acc = 0;
        uint32_t acc_phase = 0;
        volatile uint32_t* abort_flag = misc + 1;
        Cursor cur(tab, args);
        TileInfo ti;
        for (int L = pair; cur.at(args, args_dn, L, ti); L += npairs) {
            const bool gu = MODE == MODE_GATEUP || (MODE == MODE_FUSED && ti.mode == 0);
            const GemmArgs& A = (MODE == MODE_FUSED && ti.mode == 1) ? args_dn : args;
            const bool ok = mbar_wait(tfull_bar(acc), acc_phase, args.err, DEV_ERR_TIMEOUT_EPILOGUE);
            if (gu) {
                // the 4 warps of a half meet at named barriers below: leave together or not at all
                if (!__all_sync(0xffffffffu, ok) && lane == 0) *abort_flag = 1u;
                named_bar_sync(bar_id, 128);
                if (*abort_flag) break;
            } else {
                if (!__all_sync(0xffffffffu, ok)) break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * 256u;
            using OT = typename GemmAct<ET, FP8W>::type;  // hidden rows (gate/up's output)
            OT* outp = reinterpret_cast<OT*>(ti.shared ? A.out_shared : A.out_routed);
            const long long ld = ti.shared ? A.ld_shared : A.ld_routed;
            const int32_t* rowmap = ti.shared ? A.rowmap_shared : A.rowmap_routed;
            const float* colscale = ti.shared ? A.colscale_shared : A.colscale_routed;
            // coded weights: the scale of this TMEM lane's weight column (lane =
            // row of the A tile: gate/up [gate 64 | up 64] features, down 128)
            float wsc = 1.0f;
            if constexpr (WSC) {
                const int r = q * 32 + lane;
                const int f = gu ? ti.f0 + 64 * (int)rank + (r & 63) : ti.f0 + 128 * (int)rank + r;
                const int wcol = (gu && r >= 64) ? ti.up_off + f : f;
                wsc = f < ti.M ? A.wscale[ti.expert][wcol] : 0.0f;
            }
            if (A.partial_out) {
                // split-K: store this split's fp32 partial; row = slot (gate/up) or
                // token (down), column = the weight column of this TMEM lane
                float* pbase = ti.shared ? A.part_shared : A.part_routed;
                const long long pld = ti.shared ? A.ld_part_shared : A.ld_part_routed;
                const long long pst = ti.shared ? A.part_stride_shared : A.part_stride_routed;
                float* pp = pbase + pst * ti.split;
                int col, fcheck;
                if (gu) {
                    const int r = q * 32 + lane;                      // 0..127: [gate 64 | up 64]
                    fcheck = ti.f0 + 64 * (int)rank + (r & 63);       // feature
                    col = (r < 64 ? 0 : ti.up_off) + fcheck;
                } else {
                    fcheck = ti.f0 + 128 * (int)rank + q * 32 + lane;
                    col = fcheck;
                }
                const bool fvalid = fcheck < ti.M;
                // down: a token row's scale (the FP8 activation mode's hidden
                // row scale) applies here; gate/up partials take theirs in the finish
                const float* tscale = !gu ? (ti.shared ? A.colscale_shared : A.colscale_routed)
                                                        : nullptr;
                for (int c = 32 * half; c < ti.n_valid; c += CSTEP) {
                    const bool cval = c + lane < ti.n_valid;
                    const int my_row =
                        cval ? (rowmap ? rowmap[ti.row0 + c + lane] : ti.row0 + c + lane) : 0;
                    const float my_ts = (cval && tscale) ? tscale[ti.row0 + c + lane] : 1.0f;
                    float v[32];
                    tmem_ld_32x32(tb + (uint32_t)c, v);
                    tmem_wait_ld();
                    if constexpr (WSC) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= wsc;
                    }
                    if constexpr (ACT8) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= __shfl_sync(0xffffffffu, my_ts, i);
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int orow = __shfl_sync(0xffffffffu, my_row, i);
                        if (fvalid && c + i < ti.n_valid) pp[(size_t)orow * pld + col] = v[i];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));
                if (++acc == Cfg::ACC_BUFS) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
                continue;
            }
            for (int c = 32 * half; c < ti.n_valid; c += CSTEP) {
                // output row (token or slot) and scale of each of the 32 columns, one per lane
                const bool cval = c + lane < ti.n_valid;
                const int my_row =
                    cval ? (rowmap ? rowmap[ti.row0 + c + lane] : ti.row0 + c + lane) : 0;
                const float my_scale = (cval && colscale) ? colscale[ti.row0 + c + lane] : 1.0f;
                float v[32];
                tmem_ld_32x32(tb + (uint32_t)c, v);
                tmem_wait_ld();
                if constexpr (WSC) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= wsc;
                }
                if (gu) {
                    // lanes 0-63: gate rows, 64-127: up rows of the same 64 features.
                    // Gate warps (q 0,1) finish columns c..c+15, up warps (q 2,3)
                    // columns c+16..c+31; each hands the other half over.
                    const bool gate_warp = q < 2;
                    const int pq = q & 1;  // feature quarter of the pair
                    float* xg = xch_h + (0 * 2 + pq) * 32 * Cfg::XLD;  // gate values, cols 16..31
                    float* xu = xch_h + (1 * 2 + pq) * 32 * Cfg::XLD;  // up values, cols 0..15
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (gate_warp) xg[lane * Cfg::XLD + i] = v[16 + i];
                        else xu[lane * Cfg::XLD + i] = v[i];
                    }
                    named_bar_sync(bar_id, 128);
                    const int f = ti.f0 + 64 * (int)rank + 32 * pq + lane;
                    const bool fvalid = f < ti.M;
                    const int cb = gate_warp ? 0 : 16;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int col = cb + i;
                        const int orow = __shfl_sync(0xffffffffu, my_row, col);
                        const float g = __shfl_sync(0xffffffffu, my_scale, col);
                        const float gv = gate_warp ? v[i] : xg[lane * Cfg::XLD + i];
                        const float uv = gate_warp ? xu[lane * Cfg::XLD + i] : v[16 + i];
                        const float hv = silu_f(g * gv) * (g * uv);
                        if constexpr (FP8W) {  // hidden rows held in f16: report values beyond its range
                            if (fvalid && c + col < ti.n_valid && !(fabsf(hv) < 65520.0f))  // rounds to inf
                                atomicOr(A.err, DEV_ERR_F16_RANGE);
                        }
                        if (fvalid && c + col < ti.n_valid)
                            store_elem(outp + (size_t)orow * ld + f, hv);
                    }
                    named_bar_sync(bar_id, 128);  // exchange buffer free for the next chunk
                } else {
                    const int f = ti.f0 + 128 * (int)rank + 32 * q + lane;
                    const bool fvalid = f < ti.M;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int orow = __shfl_sync(0xffffffffu, my_row, i);
                        if (fvalid && c + i < ti.n_valid)
                            store_elem(outp + (size_t)orow * ld + f, v[i]);
                    }
                }
            }
            if constexpr (MODE == MODE_FUSED) {
                if (gu) {  // this warp's hidden values of the tile are stored: count them
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) atomicAdd(args.done + (ti.shared ? 0 : 1), 1u);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(mapa_shared(tempty_bar(acc), 0));  // to the leader
            if (++acc == Cfg::ACC_BUFS) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncwarp();
    cluster_sync();  // no CTA of the pair leaves while the other may still use its memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace l4moe
