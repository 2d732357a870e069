// moe_gemm.cuh -- persistent grouped GEMM on the 5th-generation tensor cores
// (tcgen05 + TMEM accumulators + TMA-fed shared-memory pipeline) for the
// three contractions of the layer:
//
//   gate/up  : a = g * (x . W_gate_up)  then h = silu(a[:F]) * a[F:]
//              (SwiGLU), for the shared expert (g = 1) and every routed
//              expert (x rows in expert order, g = the token's sigmoid gate,
//              applied to the fp32 accumulator: the gate scales the input
//              and the contraction is linear in it) in one launch
//   down     : out[token] = h_shared . Ws_down + h_routed . W_down[e], both
//              contractions accumulated into one TMEM tile (a shared K segment
//              then the routed one), so the sum is rounded once
//
// llm-architectures-explained "Llama 4 Maverick", field table rows
// ffns.moe.gated / d_expert / d_shared: every expert and the shared expert is
// a gated MLP of width 8192; superteams.ai "Llama 4" glossary, routing
// sketch: the layer output is the shared expert's output plus the routed
// expert's.
//
// Orientation ("swap-AB"): the weight is the MMA A operand (M = 128 output
// features, read MN-major straight from the row-major [K, N] weight) and the
// activations are the B operand (N = up to 256 tokens, K-major rows).  A
// group's token count is only padded to a multiple of 16, so ragged experts
// (and decode, T <= 128) waste little tensor work.  For gate/up a tile holds
// the gate block and the matching up block of 128 features each, as two TMEM
// accumulators, so the SwiGLU is computed in the epilogue from registers.
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads into a STAGES-deep ring
// of shared-memory stages; warp 1 owns TMEM (alloc/dealloc) and lane 0
// issues the MMAs and commits; warps 2..5 are the epilogue (warp w reads TMEM
// lanes 32*(w%4) .. +31).  Every mbarrier wait is bounded; on a timeout a
// role records a bit in the error word and returns, the producer drains its
// in-flight copies, the MMA thread waits for its issued MMAs, and TMEM is
// freed before exit.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "permute.cuh"
#include "ptx.cuh"

namespace l4moe {

enum GemmMode : int { MODE_GATEUP = 0, MODE_DOWN = 1 };

template <typename ET>
struct ElemCfg;
template <>
struct ElemCfg<__nv_bfloat16> {
    static constexpr int BYTES = 2;
    static constexpr int BK = 64;     // K elements per stage (one 128-byte row)
    static constexpr int MMA_K = 16;  // K per tcgen05.mma (kind::f16)
    static constexpr uint32_t FMT = 1;
    static constexpr uint32_t A_LAYOUT = 2;   // MN-major weights: 128B swizzle, 16B unit
    static constexpr uint32_t A_SBO = 1024;   // 8 K rows per atom
};
template <>
struct ElemCfg<float> {
    static constexpr int BYTES = 4;
    static constexpr int BK = 32;
    static constexpr int MMA_K = 8;   // kind::tf32
    static constexpr uint32_t FMT = 2;
    static constexpr uint32_t A_LAYOUT = 1;   // MN-major 32-bit: 128B swizzle, 32B unit
    static constexpr uint32_t A_SBO = 512;    // 4 K rows per atom
};

struct GemmArgs {
    const GroupTable* table;
    const CUtensorMap* a_maps;  // weights, [E + 1]: routed experts then the shared expert
    int num_experts;            // E (expert index E = shared)
    int k_routed, k_shared;     // main K segment per class (gate/up: d, d; down: F)
    int k_pre;                  // down: leading K segment over the shared expert (Fs), else 0
    int m_routed, m_shared;     // output features per class (F / Fs, or d)
    int up_routed, up_shared;   // gate/up: column offset of the "up" half (F / Fs)
    void* out_routed;
    long long ld_routed;
    void* out_shared;
    long long ld_shared;
    const int32_t* rowmap_routed;  // down: output row of a slot (perm), else null
    const int32_t* rowmap_shared;  // gate/up: slot of a token (inv), else null
    const float* colscale_routed;  // gate/up: sigmoid gate of each slot, else null
    unsigned* err;
};

template <int MODE, typename ET>
struct GemmCfg {
    using C = ElemCfg<ET>;
    static constexpr int A_OPS = (MODE == MODE_GATEUP) ? 2 : 1;
    static constexpr int A_OP_BYTES = kFeatTile * 128;               // 128 features x 128 B of K
    static constexpr int A_BOX_FEATS = 128 / C::BYTES;               // features per A box
    static constexpr int A_BOXES = kFeatTile / A_BOX_FEATS;          // boxes per A operand
    static constexpr int A_BOX_BYTES = C::BK * 128;                  // BK rows x 128 B
    static constexpr int B_BOX_ROWS = 64;
    static constexpr int B_BOX_BYTES = B_BOX_ROWS * 128;
    static constexpr int B_BYTES = kTokTile * 128;
    static constexpr int STAGE_BYTES = A_OPS * A_OP_BYTES + B_BYTES;
    static constexpr int STAGES = (MODE == MODE_GATEUP) ? 3 : 4;
    static constexpr int ACC_BUFS = (MODE == MODE_GATEUP) ? 1 : 2;  // 512 TMEM columns either way
    static constexpr int TMEM_COLS = 512;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * 2 + 1;
    static constexpr size_t SMEM_BYTES =
        1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES + NUM_BARS * 8 + 16 +
        sizeof(GroupTable);
};

struct TileInfo {
    int expert, row0, n_valid, n_mma, f0, K, k_pre, M, up_off;
    bool shared;
};

__device__ __forceinline__ TileInfo decode_tile(const GroupTable& tab, const GemmArgs& a, int L) {
    int lo = 0, hi = tab.num_groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab.tile_start[mid] <= L) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int local = L - tab.tile_start[g];
    const int rows = tab.rows[g];
    const int ntb = (rows + kTokTile - 1) / kTokTile;
    const int tb = local % ntb;
    const int fb = local / ntb;
    TileInfo ti;
    ti.expert = tab.expert[g];
    ti.shared = (ti.expert == a.num_experts);
    ti.row0 = tab.row0[g] + tb * kTokTile;
    ti.n_valid = min(kTokTile, rows - tb * kTokTile);
    ti.n_mma = (ti.n_valid + 15) & ~15;
    ti.f0 = fb * kFeatTile;
    ti.k_pre = ti.shared ? 0 : a.k_pre;
    ti.K = ti.k_pre + (ti.shared ? a.k_shared : a.k_routed);
    ti.M = ti.shared ? a.m_shared : a.m_routed;
    ti.up_off = ti.shared ? a.up_shared : a.up_routed;
    return ti;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <int MODE, typename ET>
__global__ void __launch_bounds__(192, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap b_routed,
                    const __grid_constant__ CUtensorMap b_shared, const GemmArgs args) {
    using Cfg = GemmCfg<MODE, ET>;
    using C = ElemCfg<ET>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)Cfg::STAGES * Cfg::STAGE_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
    GroupTable* tab = reinterpret_cast<GroupTable*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t stage0 = smem_u32(smem);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (Cfg::STAGES + s); };
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * Cfg::STAGES + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * Cfg::STAGES + 4);

    // work list -> shared memory
    {
        const int* src = reinterpret_cast<const int*>(args.table);
        int* dst = reinterpret_cast<int*>(tab);
        for (int i = threadIdx.x; i < (int)(sizeof(GroupTable) / 4); i += blockDim.x) dst[i] = src[i];
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
        }
        mbar_init(drain_bar, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&b_routed);
        tma_prefetch_desc(&b_shared);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tab->total_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t used = 0, last_par = 0;  // per-stage: issued at least once / parity
            for (int L = blockIdx.x; L < total; L += gridDim.x) {
                const TileInfo ti = decode_tile(*tab, args, L);
                const CUtensorMap* amap_main = args.a_maps + ti.expert;
                const CUtensorMap* amap_pre = args.a_maps + args.num_experts;
                const void* bmap_main = ti.shared ? (const void*)&b_shared : (const void*)&b_routed;
                const int nkb = ti.K / C::BK;
                const int nkb_pre = ti.k_pre / C::BK;
                const int nbb = (ti.n_mma + Cfg::B_BOX_ROWS - 1) / Cfg::B_BOX_ROWS;
                const uint32_t tx =
                    Cfg::A_OPS * Cfg::A_OP_BYTES + (uint32_t)nbb * Cfg::B_BOX_BYTES;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, args.err, DEV_ERR_TIMEOUT_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar(stage), tx);
                    const uint32_t sb = stage0 + (uint32_t)stage * Cfg::STAGE_BYTES;
                    // leading shared-expert segment (down only), then the tile's own weights
                    const bool pre = kb < nkb_pre;
                    const CUtensorMap* amap = pre ? amap_pre : amap_main;
                    const void* bmap = pre ? (const void*)&b_shared : bmap_main;
                    const int k = (pre ? kb : kb - nkb_pre) * C::BK;
#pragma unroll
                    for (int op = 0; op < Cfg::A_OPS; ++op) {
                        const int col0 = (op == 0 ? 0 : ti.up_off) + ti.f0;
#pragma unroll
                        for (int bx = 0; bx < Cfg::A_BOXES; ++bx)
                            tma_load_2d(sb + op * Cfg::A_OP_BYTES + bx * Cfg::A_BOX_BYTES, amap,
                                        full_bar(stage), col0 + bx * Cfg::A_BOX_FEATS, k);
                    }
                    const uint32_t bb = sb + Cfg::A_OPS * Cfg::A_OP_BYTES;
                    for (int j = 0; j < nbb; ++j)
                        tma_load_2d(bb + j * Cfg::B_BOX_BYTES, bmap, full_bar(stage), k,
                                    ti.row0 + j * Cfg::B_BOX_ROWS);
                    used |= 1u << stage;
                    last_par = (last_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // drain: every issued copy must land before the CTA may exit
            for (int s = 0; s < Cfg::STAGES; ++s)
                if (used & (1u << s))
                    mbar_wait(full_bar(s), (last_par >> s) & 1u, args.err, DEV_ERR_TIMEOUT_PRODUCER);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int L = blockIdx.x; L < total; L += gridDim.x) {
                const TileInfo ti = decode_tile(*tab, args, L);
                if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, args.err, DEV_ERR_TIMEOUT_MMA)) break;
                tc_fence_after();
                const uint32_t idesc = make_idesc(C::FMT, 1u, 0u, (uint32_t)ti.n_mma, 128u);
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * 256u;
                const int nkb = ti.K / C::BK;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, args.err, DEV_ERR_TIMEOUT_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sb = stage0 + (uint32_t)stage * Cfg::STAGE_BYTES;
                    const uint32_t bb = sb + Cfg::A_OPS * Cfg::A_OP_BYTES;
#pragma unroll
                    for (int kk = 0; kk < C::BK / C::MMA_K; ++kk) {
                        const uint64_t bdesc = smem_desc(bb + kk * 32, 16, 1024, 2);
#pragma unroll
                        for (int op = 0; op < Cfg::A_OPS; ++op) {
                            const uint64_t adesc =
                                smem_desc(sb + op * Cfg::A_OP_BYTES + kk * C::MMA_K * 128,
                                          Cfg::A_BOX_BYTES, C::A_SBO, C::A_LAYOUT);
                            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                            if constexpr (C::FMT == 1)
                                mma_bf16(d_tmem + op * 256u, adesc, bdesc, idesc, accum);
                            else
                                mma_tf32(d_tmem + op * 256u, adesc, bdesc, idesc, accum);
                        }
                    }
                    mma_commit(empty_bar(stage));
                    if (++stage == Cfg::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(tfull_bar(acc));
                if (++acc == Cfg::ACC_BUFS) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // every issued MMA must finish before TMEM is released
            mma_commit(drain_bar);
            mbar_wait(drain_bar, 0, args.err, DEV_ERR_TIMEOUT_MMA);
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;            // TMEM lane quarter of this warp
        const int row = q * 32 + lane;     // feature within the tile
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int L = blockIdx.x; L < total; L += gridDim.x) {
            const TileInfo ti = decode_tile(*tab, args, L);
            // warp-uniform outcome: the TMEM loads below are .sync.aligned
            const bool ok = mbar_wait(tfull_bar(acc), acc_phase, args.err, DEV_ERR_TIMEOUT_EPILOGUE);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int f = ti.f0 + row;
            const bool fvalid = f < ti.M;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * 256u;
            ET* outp = reinterpret_cast<ET*>(ti.shared ? args.out_shared : args.out_routed);
            const long long ld = ti.shared ? args.ld_shared : args.ld_routed;
            const int32_t* rowmap = ti.shared ? args.rowmap_shared : args.rowmap_routed;
            const float* colscale = ti.shared ? nullptr : args.colscale_routed;
            for (int c = 0; c < ti.n_valid; c += 32) {
                // output row (token or slot) and scale of each of the 32 columns, one per lane
                const bool cval = c + lane < ti.n_valid;
                const int my_row =
                    cval ? (rowmap ? rowmap[ti.row0 + c + lane] : ti.row0 + c + lane) : 0;
                const float my_scale = (cval && colscale) ? colscale[ti.row0 + c + lane] : 1.0f;
                float v[32];
                tmem_ld_32x32(tb + (uint32_t)c, v);
                if constexpr (MODE == MODE_GATEUP) {
                    float u[32];
                    tmem_ld_32x32(tb + 256u + (uint32_t)c, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int orow = __shfl_sync(0xffffffffu, my_row, i);
                        const float g = __shfl_sync(0xffffffffu, my_scale, i);
                        if (fvalid && c + i < ti.n_valid)
                            store_elem(outp + (size_t)orow * ld + f, silu_f(g * v[i]) * (g * u[i]));
                    }
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int orow = __shfl_sync(0xffffffffu, my_row, i);
                        if (fvalid && c + i < ti.n_valid)
                            store_elem(outp + (size_t)orow * ld + f, v[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(acc));
            if (++acc == Cfg::ACC_BUFS) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace l4moe
