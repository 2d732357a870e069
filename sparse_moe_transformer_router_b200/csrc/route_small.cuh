// route_small.cuh -- the whole routing of a small batch (decode) in one
// launch: the router logits, the top-k selection with its sigmoid gates, the
// per-expert histogram, scan and stable slots, the GEMM work lists and the
// copy of the input rows into expert order.
//
// superteams.ai "Llama 4" glossary, section "Mixture of Experts: Why Total
// and Active Parameters Diverge" (routing sketch): every expert gets one
// score per token and the token goes to the best one; KerasFormers "Llama
// 4", "What is unusual about the block": the chosen expert is reached
// through a sigmoid gate on its input.
//
// With a few tokens the router is a matrix-vector product bound by reading
// W_router (d x E, 1.3 MB for Maverick), and everything after it is a chain
// of short dependent steps.  As separate kernels (router, permutation, row
// copy) the chain costs several launches and global-memory round trips.
// Here one cluster of kSmallCluster CTAs does it all: CTA z streams its
// share of the rows of W_router (64-row chunks, contiguous, through a double
// buffer in shared memory: the next chunk's loads are in flight while the
// current one is used) and keeps partial logits for all T tokens; rank 0
// adds the ranks' partials in rank order (deterministic) through distributed
// shared memory, adds the bias and does the rest alone while the others
// exit.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <type_traits>

#include "permute.cuh"
#include "ptx.cuh"
#include "router.cuh"
#include "schedule.cuh"
#include "topk.cuh"

namespace l4moe {

constexpr int kSmallMaxTokens = 16;  // batches up to this size take this kernel
constexpr int kSmallCluster = 8;     // CTAs (one cluster) sharing the rows of W_router
constexpr int kSmallChunk = 64;      // W_router rows per shared-memory chunk
constexpr int kSmallThreads = 256;
constexpr int kSmallMaxEntries = kSmallMaxTokens * kMaxTopK;
constexpr int kSmallStageVec = 16;   // 16-byte vectors per thread per chunk (64 rows x 256 x fp32)

// Rows of W_router CTA z of the cluster takes: 64-row chunks [c0, c1).
__host__ __device__ inline void small_chunks(int d, int z, int& c0, int& c1) {
    const int n = d / kSmallChunk;
    c0 = (n * z) / kSmallCluster;
    c1 = (n * (z + 1)) / kSmallCluster;
}

// Dynamic shared memory: the x rows of the CTA's chunks [T][rows] fp32, two
// W_router chunk buffers [64][E] in its storage type, then the partial
// logits [T][E] fp32 (aliasing the first buffer once the loop is done) --
// also rank 0's logits.
template <typename ET>
__host__ __device__ constexpr size_t route_small_smem_bytes(int T, int E, int d) {
    const int n = d / kSmallChunk;
    const size_t rows = (size_t)((n + kSmallCluster - 1) / kSmallCluster) * kSmallChunk;
    const size_t wbuf = sizeof(ET) * (size_t)kSmallChunk * E;
    const size_t part = sizeof(float) * (size_t)T * E;
    return sizeof(float) * (size_t)T * rows + 2 * (wbuf > part ? wbuf : part);
}

// Grid (1, 1, kSmallCluster), launched as one cluster along z.  GT: the GEMMs'
// activation type (the layer's, or f16 for 8- or 4-bit weights; x16 then
// receives x in f16, token order, each row divided by its power-of-two scale,
// recorded in tokscale and folded into gslot).
template <typename ET, typename GT>
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(
    const ET* __restrict__ x, const ET* __restrict__ Wr, const float* __restrict__ bias, int T, int d,
    int E, int k, int32_t* __restrict__ idx, float* __restrict__ gate, float* __restrict__ lmax,
    float* __restrict__ margin, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, float* __restrict__ gslot, GroupTable* tab_gu,
    GroupTable* tab_dn, int fb_gu_routed, int fb_gu_shared, int fb_down, GT* __restrict__ xg,
    GT* __restrict__ x16, float* __restrict__ tokscale) {
    pdl_enter();
    extern __shared__ __align__(16) uint8_t rs_smem[];
    __shared__ int32_t s_ent[kSmallMaxEntries];   // selected expert of entry n = t * k + j
    __shared__ int32_t s_rank[kSmallMaxEntries];  // rank of the entry inside its expert
    __shared__ float s_gate[kSmallMaxEntries];
    __shared__ int32_t s_rows[kMaxGroups];        // entries per expert
    __shared__ int32_t s_off[kMaxGroups + 1];     // exclusive prefix of s_rows
    __shared__ float s_scale[kSmallMaxTokens];    // power-of-two row scale (f16 rows; else 1)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t z = cluster_ctarank();

    int c0, c1;
    small_chunks(d, (int)z, c0, c1);
    const int nrows = (c1 - c0) * kSmallChunk;
    const int maxrows = ((d / kSmallChunk + kSmallCluster - 1) / kSmallCluster) * kSmallChunk;
    float* xs = reinterpret_cast<float*>(rs_smem);  // [T][maxrows]
    const size_t wbuf = sizeof(ET) * (size_t)kSmallChunk * E;
    const size_t pbytes = sizeof(float) * (size_t)T * E;
    const size_t buf = wbuf > pbytes ? wbuf : pbytes;
    uint8_t* const wb0 = rs_smem + sizeof(float) * (size_t)T * maxrows;
    uint8_t* const wb1 = wb0 + buf;
    float* part = reinterpret_cast<float*>(wb0);  // [T][E] once the chunks are done

    // ---------------------------------------------- partial logits of this CTA's rows
    // a chunk of W_router is kSmallChunk * E contiguous elements: 16-byte
    // vectors, at most kSmallStageVec per thread
    const int nvec = (int)(wbuf / 16);
    auto fetch = [&](int c, uint4 (&r)[kSmallStageVec]) {
        const uint4* src = reinterpret_cast<const uint4*>(Wr + (size_t)c * kSmallChunk * E);
#pragma unroll
        for (int q = 0; q < kSmallStageVec; ++q) {
            const int i = tid + kSmallThreads * q;
            if (i < nvec) r[q] = src[i];
        }
    };
    auto stash = [&](uint8_t* dst, const uint4 (&r)[kSmallStageVec]) {
#pragma unroll
        for (int q = 0; q < kSmallStageVec; ++q) {
            const int i = tid + kSmallThreads * q;
            if (i < nvec) reinterpret_cast<uint4*>(dst)[i] = r[q];
        }
    };
    uint4 stage[kSmallStageVec];
    if (c1 > c0) fetch(c0, stage);
    {
        const int V = 16 / (int)sizeof(ET);
        const int xv = nrows / V;  // the x columns of this CTA's rows, 16-byte vectors
        for (int i = tid; i < T * xv; i += kSmallThreads) {
            const int t = i / xv, c = i - t * xv;
            ET tmp[16 / sizeof(ET)];
            *reinterpret_cast<uint4*>(tmp) =
                reinterpret_cast<const uint4*>(x + (size_t)t * d + (size_t)c0 * kSmallChunk)[c];
#pragma unroll
            for (int u = 0; u < V; ++u) xs[t * maxrows + c * V + u] = to_f32(tmp[u]);
        }
    }
    // thread -> (expert e, token group g); a group takes tokens g, g + G, ...
    const int G = max(1, kSmallThreads / E);
    const int e = tid % E, g = tid / E;
    const bool active = g < G && tid < G * E;
    float acc[kSmallMaxTokens];
#pragma unroll
    for (int j = 0; j < kSmallMaxTokens; ++j) acc[j] = 0.f;
    for (int c = c0; c < c1; ++c) {
        uint8_t* cur = ((c - c0) & 1) ? wb1 : wb0;
        stash(cur, stage);
        __syncthreads();                  // chunk c in shared memory (and the x rows, first time)
        if (c + 1 < c1) fetch(c + 1, stage);  // in flight while chunk c is used
        if (active) {
            const ET* wcol = reinterpret_cast<const ET*>(cur) + e;
            const int r0 = (c - c0) * kSmallChunk;
#pragma unroll 4
            for (int kk = 0; kk < kSmallChunk; ++kk) {
                const float w = to_f32(wcol[kk * E]);
#pragma unroll
                for (int j = 0; j < kSmallMaxTokens; ++j) {
                    const int t = g + j * G;
                    if (t < T) acc[j] = fmaf(xs[t * maxrows + r0 + kk], w, acc[j]);
                }
            }
        }
        __syncthreads();                  // buffer free for chunk c + 2
    }
    if (active) {
#pragma unroll
        for (int j = 0; j < kSmallMaxTokens; ++j) {
            const int t = g + j * G;
            if (t < T) part[t * E + e] = acc[j];
        }
    }
    // (every (token, expert) entry has one active thread: CTAs without rows write zeros)
    cluster_sync();  // every rank's partial complete in its shared memory
    if (z != 0) {
        cluster_sync();  // rank 0 has read it: leave
        return;
    }

    // ---------------------------------------------- rank 0: logits = ranks' partials in order, + bias
    float* lg = part;
    {
        const int n4 = (T * E) / 4;  // E * T may not be a multiple of 4: the tail below
        for (int i = tid; i < n4; i += kSmallThreads) {
            float4 r[kSmallCluster - 1];
#pragma unroll
            for (int zz = 1; zz < kSmallCluster; ++zz)
                r[zz - 1] = ld_shared_cluster_v4(mapa_shared(smem_u32(part + 4 * i), (uint32_t)zz));
            float4 v = reinterpret_cast<float4*>(part)[i];
#pragma unroll
            for (int zz = 0; zz < kSmallCluster - 1; ++zz) {
                v.x += r[zz].x;
                v.y += r[zz].y;
                v.z += r[zz].z;
                v.w += r[zz].w;
            }
            reinterpret_cast<float4*>(lg)[i] = v;
        }
        for (int i = 4 * n4 + tid; i < T * E; i += kSmallThreads) {
            float v = part[i];
            for (int zz = 1; zz < kSmallCluster; ++zz)
                v += ld_shared_cluster_f32(mapa_shared(smem_u32(part + i), (uint32_t)zz));
            lg[i] = v;
        }
    }
    cluster_sync();  // the other ranks may leave
    for (int i = tid; i < T * E; i += kSmallThreads) lg[i] += bias ? bias[i % E] : 0.f;
    __syncthreads();

    // ---------------------------------------------- top-k, one warp per token
    // each lane keeps the list of its experts (lane, lane + 32, ...: ascending,
    // so ties keep the lower index), then k + 1 butterfly rounds each take
    // the first head in (value, index) order
    for (int t = warp; t < T; t += kSmallThreads / 32) {
        TopK tk;
        tk.init();
        for (int ee = lane; ee < E; ee += 32) tk.offer(lg[t * E + ee], ee);
        TopK sel;
        sel.init();
        int pos = 0;
#pragma unroll
        for (int j = 0; j <= kMaxTopK; ++j) {
            float hv = tk.value(pos);
            int hi = pos <= kMaxTopK ? tk.index(pos) : -1;
            int hl = lane;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
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
            if (hl == lane && hi >= 0) ++pos;
        }
        if (lane == 0) {
            sel.fill_empty(k);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < k) {
                    const int n = t * k + j;
                    const float gv = 1.0f / (1.0f + expf(-sel.value(j)));
                    idx[n] = sel.index(j);
                    lmax[n] = sel.value(j);
                    gate[n] = gv;
                    s_ent[n] = sel.index(j);
                    s_gate[n] = gv;
                }
            }
            margin[t] = sel.value(k - 1) - sel.value(k);
        }
    }
    for (int ee = tid; ee < E; ee += kSmallThreads) s_rows[ee] = 0;
    // each token row's power-of-two scale into f16's range (coded-weight
    // layers, f16_row_scale), one warp per token
    const int nv = d * (int)sizeof(ET) / 16;
    for (int t = warp; t < T; t += kSmallThreads / 32) {
        float sc = 1.0f;
        if constexpr (!std::is_same<ET, GT>::value) {
            float m = 0.0f;
            for (int i = lane; i < nv; i += 32) m = absmax_vec(reinterpret_cast<const uint4*>(x + (size_t)t * d)[i], m);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            sc = f16_row_scale(m);
            if (lane == 0 && tokscale) tokscale[t] = sc;
        }
        if (lane == 0) s_scale[t] = sc;
    }
    __syncthreads();

    // ---------------------------------------------- ranks, counts, offsets (warp 0)
    const int Tv = T * k;
    if (warp == 0) {
        for (int n0 = 0; n0 < Tv; n0 += 32) {
            const int n = n0 + lane;
            const int ee = n < Tv ? s_ent[n] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, ee);
            const int below = __popc(peers & ((1u << lane) - 1u));
            if (ee >= 0) s_rank[n] = s_rows[ee] + below;  // entries of ee before this chunk, then this chunk's
            __syncwarp();
            if (ee >= 0 && below == 0) s_rows[ee] += __popc(peers);
            __syncwarp();
        }
        int local[8];
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int ee = lane * 8 + j;
            local[j] = ee < E ? s_rows[ee] : 0;
            sum += local[j];
        }
        const int incl = warp_incl_scan(sum);
        int a = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int ee = lane * 8 + j;
            if (ee < E) {
                s_off[ee] = a;
                offsets[ee] = a;
                counts[ee] = local[j];
            }
            a += local[j];
        }
        if (lane == 31) {
            s_off[E] = incl;
            offsets[E] = incl;
        }
    }
    __syncthreads();
    for (int n = tid; n < Tv; n += kSmallThreads) {
        const int slot = s_off[s_ent[n]] + s_rank[n];
        inv[n] = slot;
        perm[slot] = n;
        gslot[slot] = s_gate[n] * s_scale[n / k];
    }
    if (warp == 0) {
        // gate/up: candidate 0 is the shared expert, 1..E the routed experts
        build_table(
            tab_gu, E + 1, [&](int gg) { return gg == 0 ? T : s_rows[gg - 1]; },
            [&](int gg) { return gg == 0 ? 0 : s_off[gg - 1]; }, [&](int gg) { return gg == 0 ? E : gg - 1; },
            [&](int gg) { return gg == 0 ? fb_gu_shared : fb_gu_routed; });
        build_table(
            tab_dn, E + 1, [&](int gg) { return gg == 0 ? T : s_rows[gg - 1]; },
            [&](int gg) { return gg == 0 ? 0 : s_off[gg - 1]; }, [&](int gg) { return gg == 0 ? E : gg - 1; },
            [&](int) { return fb_down; });
    }

    // ---------------------------------------------- rows in expert order
    // xg[slot of n] = x[n / k] (16-byte vectors, converted for coded-weight
    // layers), and x16[t] = x[t] in token order when it is given
    const int rows = Tv + (x16 ? T : 0);
    for (int i = tid; i < rows * nv; i += kSmallThreads) {
        const int r = i / nv, c = i - r * nv;
        const bool tok = r >= Tv;
        const int t = tok ? r - Tv : r / k;
        const int orow = tok ? t : s_off[s_ent[r]] + s_rank[r];
        const uint4 v = cvt_row_vec(reinterpret_cast<const uint4*>(x + (size_t)t * d)[c], ET{}, GT{},
                                    1.0f / s_scale[t]);
        reinterpret_cast<uint4*>((tok ? x16 : xg) + (size_t)orow * d)[c] = v;
    }
}

}  // namespace l4moe
