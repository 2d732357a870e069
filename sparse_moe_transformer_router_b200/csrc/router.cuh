// router.cuh -- router logits, top-1 selection and the sigmoid gate.
//
// superteams.ai "Llama 4" glossary, section "Mixture of Experts: Why Total
// and Active Parameters Diverge": the router scores every expert once per
// token and the token goes to the single best one.  KerasFormers "Llama 4",
// section "What is unusual about the block": the chosen expert is reached
// through a sigmoid gate on its input.
//
// Two routers: the tensor-core one further down (bf16 layers, E % 8 == 0)
// and this CUDA-core one for the others (fp32 layers, other E).
//
// One CTA handles TT = NT / TPT tokens; TPT threads share a token and each
// owns NG groups of 4 consecutive experts.  x and W_router are staged through
// shared memory in K chunks of 64 and converted to fp32; each thread keeps
// 4 * NG fp32 accumulators (sequential fma over k).  Each thread offers its
// experts, in ascending order, to its own top-k list (a strict ">" keeps the
// lower index first among equal values; NaN is never taken); the token's TPT
// threads then take k + 1 heads in (value, then index) order with butterfly
// shuffles -- the sequential rule "the k largest, lowest index first among
// equal values", whose k = 1 case is the arg-max.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "topk.cuh"

namespace l4moe {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int kRouterKC = 64;

template <typename ET>
struct Vec16;
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ static void load(const float* p, float* out) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x, out[1] = v.y, out[2] = v.z, out[3] = v.w;
    }
};
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const __nv_bfloat16* p, float* out) {
        const uint4 v = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            out[2 * i] = __uint_as_float(w[i] << 16);
            out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

// Dynamic shared memory of router_kernel<ET, NT, TPT, NG>.
template <int NT, int TPT, int NG>
constexpr size_t router_smem_bytes() {
    return sizeof(float) * ((NT / TPT) * (kRouterKC + 1) + kRouterKC * 4 * TPT * NG);
}

// NT threads; TT = NT / TPT tokens per CTA; requires d % kRouterKC == 0.
// W_router rows are loaded as 16-byte vectors when E is a multiple of the
// vector width (wr_vec), element by element otherwise.
template <typename ET, int NT, int TPT, int NG>
__global__ void __launch_bounds__(NT) router_kernel(const ET* __restrict__ x,
                                                    const ET* __restrict__ Wr,
                                                    const float* __restrict__ bias, int T, int d,
                                                    int E, int wr_vec, int32_t* __restrict__ idx,
                                                    float* __restrict__ gate,
                                                    float* __restrict__ lmax,
                                                    float* __restrict__ margin, int topk) {
    pdl_enter();
    constexpr int TT = NT / TPT;
    constexpr int EPAD = 4 * TPT * NG;
    constexpr int XLD = kRouterKC + 1;
    constexpr int V = Vec16<ET>::N;
    extern __shared__ float rsm[];
    float* xs = rsm;                  // [TT][XLD]
    float* ws = rsm + TT * XLD;       // [kRouterKC][EPAD]

    const int tid = threadIdx.x;
    const int tl = tid / TPT;         // token within the CTA
    const int r = tid % TPT;          // expert-group lane of that token
    const int t0 = blockIdx.x * TT;

    float acc[NG][4];
#pragma unroll
    for (int j = 0; j < NG; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;

    for (int kc = 0; kc < d; kc += kRouterKC) {
        for (int i = tid; i < TT * (kRouterKC / V); i += NT) {
            const int tt = i / (kRouterKC / V), k = (i % (kRouterKC / V)) * V;
            const int t = t0 + tt;
            float v[V];
            if (t < T) {
                Vec16<ET>::load(x + (size_t)t * d + kc + k, v);
            } else {
#pragma unroll
                for (int u = 0; u < V; ++u) v[u] = 0.f;
            }
#pragma unroll
            for (int u = 0; u < V; ++u) xs[tt * XLD + k + u] = v[u];
        }
        if (wr_vec) {
            const int epv = E / V;  // vectors per router row
            for (int i = tid; i < kRouterKC * epv; i += NT) {
                const int k = i / epv, e = (i % epv) * V;
                float v[V];
                Vec16<ET>::load(Wr + (size_t)(kc + k) * E + e, v);
#pragma unroll
                for (int u = 0; u < V; ++u) ws[k * EPAD + e + u] = v[u];
            }
            for (int i = tid; i < kRouterKC * (EPAD - E); i += NT) {
                const int k = i / (EPAD - E), e = E + i % (EPAD - E);
                ws[k * EPAD + e] = 0.f;
            }
        } else {
            for (int i = tid; i < kRouterKC * EPAD; i += NT) {
                const int k = i / EPAD, e = i % EPAD;
                ws[k * EPAD + e] = (e < E) ? to_f32(Wr[(size_t)(kc + k) * E + e]) : 0.f;
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kRouterKC; ++k) {
            const float xv = xs[tl * XLD + k];
#pragma unroll
            for (int j = 0; j < NG; ++j) {
                const float4 w = *reinterpret_cast<const float4*>(&ws[k * EPAD + 4 * (r + TPT * j)]);
                acc[j][0] = fmaf(xv, w.x, acc[j][0]);
                acc[j][1] = fmaf(xv, w.y, acc[j][1]);
                acc[j][2] = fmaf(xv, w.z, acc[j][2]);
                acc[j][3] = fmaf(xv, w.w, acc[j][3]);
            }
        }
        __syncthreads();
    }

    // this thread's list (its experts in ascending order)
    TopK tk;
    tk.init();
#pragma unroll
    for (int j = 0; j < NG; ++j) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int e = 4 * (r + TPT * j) + c;
            if (e < E) tk.offer(acc[j][c] + (bias ? bias[e] : 0.f), e);
        }
    }
    // the token's TPT lists (consecutive lanes): k + 1 heads in selection order
    TopK sel;
    sel.init();
    int pos = 0;  // entries of this thread's list already taken
#pragma unroll
    for (int j = 0; j <= kMaxTopK; ++j) {
        float hv = tk.value(pos);
        int hi = pos <= kMaxTopK ? tk.index(pos) : -1;
        int hl = r;
#pragma unroll
        for (int off = TPT / 2; off > 0; off /= 2) {
            const float ov = __shfl_xor_sync(0xffffffffu, hv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, hi, off);
            const int ol = __shfl_xor_sync(0xffffffffu, hl, off);
            if (topk_before(ov, oi, hv, hi)) {
                hv = ov;
                hi = oi;
                hl = ol;
            }
        }
        sel.set(j, hv, hi);
        if (hl == r && hi >= 0) ++pos;
    }
    const int t = t0 + tl;
    if (r == 0 && t < T) {
        sel.fill_empty(topk);
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < topk) {
                const size_t n = (size_t)t * topk + j;
                idx[n] = sel.index(j);
                lmax[n] = sel.value(j);
                gate[n] = 1.0f / (1.0f + expf(-sel.value(j)));
            }
        }
        margin[t] = sel.value(topk - 1) - sel.value(topk);  // k-th against the next one
    }
}

// ---------------------------------------------------------------------------
// Tensor-core router for bf16 layers with E % 8 == 0 (E <= 256), top-k
// (k = topk <= kMaxTopK; idx, gate, lmax hold [T][k], margin [T] is the k-th
// selected logit minus the next one): one CTA per
// 128-token tile computes the fp32 logits of all E experts with tcgen05 (M =
// 128 tokens, N = E rounded up to 16, K = d; x rows are the K-major A
// operand, W_router [d, E] the MN-major B operand), then each of 128 threads
// owns one token's logits in TMEM and applies the same arg-max / runner-up /
// sigmoid rule as the CUDA-core router above.  Warp 0 lane 0 issues the TMA
// loads, warp 1 lane 0 the MMAs; all four warps run the epilogue.
namespace rmma {
constexpr int STAGES = 4;
constexpr int A_BYTES = 128 * 128;     // 128 tokens x 64 K (bf16)
constexpr int B_BOX_BYTES = 64 * 128;  // 64 K rows x 64 experts (bf16)
constexpr int MAX_B_BOXES = 4;         // E <= 256
constexpr int STAGE_BYTES = A_BYTES + MAX_B_BOXES * B_BOX_BYTES;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + (2 * STAGES + 1) * 8 + 16;
// A launch whose CTAs each take n_chunk experts needs stages of the token
// tile plus ceil(n_chunk / 64) weight boxes only: fewer bytes, so that two
// CTAs fit on an SM when the experts are few.
__host__ __device__ constexpr int stage_bytes(int n_chunk) {
    return A_BYTES + ((n_chunk + 63) / 64) * B_BOX_BYTES;
}
__host__ __device__ constexpr size_t smem_bytes(int n_chunk) {
    return 1024 + (size_t)STAGES * stage_bytes(n_chunk) + (2 * STAGES + 1) * 8 + 16;
}
}  // namespace rmma

// Cluster K-split (gridDim.z = S > 1, launched as clusters of (1, 1, S)):
// CTA z of a cluster computes the partial logits of
// the same 128 tokens over K slice z and keeps them in its shared memory;
// after a cluster barrier rank 0 adds ranks 1..S-1's partials to its own in
// slice order (deterministic) and runs the arg-max epilogue.  This spreads
// the x stream of a batch of few token tiles over S times more SMs.
// Each CTA's partial (fp32, row-major [128 tokens][n_pad + 4], at most
// 130 KB for E = 256) reuses its own operand stages; rank 0 reads a token's
// row from each other rank with 16-byte loads issued before any is used.
//
// Expert-split mode (logits != null, for batches of one token tile): CTA
// (y, z) computes experts [y*n_chunk, (y+1)*n_chunk) over K slice z of
// gridDim.z; the slices meet in rank 0 of their cluster as above, which
// stores the biased fp32 logits to logits[T][E]; the arg-max then runs in
// the permutation kernel.  This spreads the router weight stream over
// (E / n_chunk) x slices SMs instead of one.
__global__ void __launch_bounds__(128, 2)
    router_mma_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap wr_map,
                      const float* __restrict__ bias, int T, int d, int E, int n_chunk,
                      float* __restrict__ logits, int32_t* __restrict__ idx,
                      float* __restrict__ gate, float* __restrict__ lmax,
                      float* __restrict__ margin, unsigned* err, int topk) {
    pdl_enter();
    extern __shared__ uint8_t rsmem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(rsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int stage_bytes = rmma::stage_bytes(n_chunk);  // this launch's stage stride
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)rmma::STAGES * stage_bytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * rmma::STAGES + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t stage0 = smem_u32(smem), bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (rmma::STAGES + s); };
    const uint32_t done_bar = bar0 + 8u * (2 * rmma::STAGES);
    const int e0 = blockIdx.y * n_chunk;        // first expert of this CTA
    const int ne = min(n_chunk, E - e0);         // experts of this CTA
    const int n_pad = (ne + 15) & ~15;
    const int nbb = (ne + 63) / 64;
    uint32_t ncols = 32;
    while ((int)ncols < n_pad) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < rmma::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(done_bar, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int t0 = blockIdx.x * 128;
    const int nkb_all = d / 64;
    const int kb_begin = (int)(((long long)nkb_all * blockIdx.z) / gridDim.z);
    const int kb_end = (int)(((long long)nkb_all * (blockIdx.z + 1)) / gridDim.z);
    const int nkb = kb_end - kb_begin;

    if (warp == 0 && lane == 0) {
        int stage = 0;
        uint32_t phase = 0, used = 0, last_par = 0;
        for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, err, DEV_ERR_TIMEOUT_PRODUCER)) break;
            mbar_arrive_expect_tx(full_bar(stage), rmma::A_BYTES + nbb * rmma::B_BOX_BYTES);
            const uint32_t sb = stage0 + (uint32_t)stage * stage_bytes;
            const int kg = (kb_begin + kb) * 64;
            tma_load_2d(sb, &x_map, full_bar(stage), kg, t0);
            tma_load_2d(sb + 64 * 128, &x_map, full_bar(stage), kg, t0 + 64);
            for (int j = 0; j < nbb; ++j)
                tma_load_2d(sb + rmma::A_BYTES + j * rmma::B_BOX_BYTES, &wr_map, full_bar(stage), e0 + 64 * j,
                            kg);
            used |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
            if (++stage == rmma::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        for (int s = 0; s < rmma::STAGES; ++s)  // drain copies in flight
            if (used & (1u << s)) mbar_wait(full_bar(s), (last_par >> s) & 1u, err, DEV_ERR_TIMEOUT_PRODUCER);
    } else if (warp == 1 && lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        const uint32_t idesc = make_idesc(1u, 0u, 1u, (uint32_t)n_pad, 128u);
        for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(full_bar(stage), phase, err, DEV_ERR_TIMEOUT_MMA)) break;
            tc_fence_after();
            const uint32_t sb = stage0 + (uint32_t)stage * stage_bytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t adesc = smem_desc(sb + kk * 32, 16, 1024, 2);
                const uint64_t bdesc = smem_desc(sb + rmma::A_BYTES + kk * 2048, rmma::B_BOX_BYTES, 1024, 2);
                mma_bf16(tmem_base, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            mma_commit(empty_bar(stage));
            if (++stage == rmma::STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        mma_commit(done_bar);  // logits complete (or every issued MMA finished)
    }
    __syncwarp();
    // epilogue: thread = token row (TMEM lane 32*warp + lane)
    const bool ok = mbar_wait(done_bar, 0, err, DEV_ERR_TIMEOUT_EPILOGUE);
    const bool kreduce = gridDim.z > 1;  // K slices: always launched as clusters along z
    const uint32_t crank = kreduce ? cluster_ctarank() : 0u;
    float* red = reinterpret_cast<float*>(smem);  // this CTA's partial, [128][n_pad + 4] (row-major)
    // K-slice partials of ranks 1..S-1: row-major [128 tokens][rld] fp32 in
    // each CTA's own (now idle) stage memory, one row per thread, so rank 0
    // reads a row with 16-byte cluster loads, all issued before they are used
    const int rld = n_pad + 4;
    if (kreduce) {
        // every CTA reaches both cluster barriers, whatever its waits gave
        if (crank != 0 && __all_sync(0xffffffffu, ok)) {
            tc_fence_after();
            float* row = red + (size_t)(32 * warp + lane) * rld;
            for (int c = 0; c < n_pad; c += 32) {
                float v[32];
                tmem_ld_32x32(tmem_base + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    if (c + i < n_pad)
                        *reinterpret_cast<float4*>(row + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
        }
        cluster_sync();  // partials of ranks 1..S-1 complete in their shared memory
    }
    // the logits of this thread's token, 32 experts at a time: own partial,
    // then slices 1..S-1 in order (a fixed order: deterministic)
    auto logits_chunk = [&](int c, float (&v)[32]) {
        tmem_ld_32x32(tmem_base + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, v);
        tmem_wait_ld();
        for (uint32_t z = 1; kreduce && z < gridDim.z; ++z) {
            const uint32_t base = mapa_shared(smem_u32(red + (size_t)(32 * warp + lane) * rld + c), z);
            float4 r[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                r[q] = (c + 4 * q < n_pad) ? ld_shared_cluster_v4(base + 16u * q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                v[4 * q] += r[q].x;
                v[4 * q + 1] += r[q].y;
                v[4 * q + 2] += r[q].z;
                v[4 * q + 3] += r[q].w;
            }
        }
    };
    if ((!kreduce || crank == 0) && __all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const int t = t0 + 32 * warp + lane;
        if (logits) {
            for (int c = 0; c < n_pad; c += 32) {
                float v[32];
                logits_chunk(c, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c + i;
                    if (e < ne && t < T) logits[(size_t)t * E + e0 + e] = v[i] + (bias ? bias[e0 + e] : 0.f);
                }
            }
        } else if (topk == 1) {
            // the arg-max (strict ">" in ascending order: the lowest index
            // among the maxima; NaN never wins) and the runner-up, branch-free
            float best = -INFINITY, second = -INFINITY;
            int bi = 0;
            for (int c = 0; c < n_pad; c += 32) {
                float v[32];
                logits_chunk(c, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c + i;
                    const float l = e < E ? v[i] + (bias ? bias[e] : 0.f) : -INFINITY;
                    const bool gt = l > best;
                    second = gt ? best : fmaxf(second, l);
                    bi = gt ? e : bi;
                    best = gt ? l : best;
                }
            }
            if (t < T) {
                idx[t] = bi;
                lmax[t] = best;
                gate[t] = 1.0f / (1.0f + expf(-best));
                margin[t] = best - second;
            }
        } else {
            TopK tk;
            tk.init();
            for (int c = 0; c < n_pad; c += 32) {
                float v[32];
                logits_chunk(c, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c + i;
                    if (e < E) tk.offer(v[i] + (bias ? bias[e] : 0.f), e);
                }
            }
            if (t < T) {
                tk.fill_empty(topk);
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) {
                    if (j < topk) {
                        const size_t n = (size_t)t * topk + j;
                        idx[n] = tk.index(j);
                        lmax[n] = tk.value(j);
                        gate[n] = 1.0f / (1.0f + expf(-tk.value(j)));
                    }
                }
                margin[t] = tk.value(topk - 1) - tk.value(topk);  // k-th against the next one
            }
        }
    }
    if (kreduce) cluster_sync();  // rank 0 done reading the others' shared memory
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, ncols);
    }
}

}  // namespace l4moe
