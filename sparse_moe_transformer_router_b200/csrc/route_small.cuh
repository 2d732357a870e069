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
// copy) the chain costs several launches and global-memory round trips; here
// the CTAs each take a slice of kSmallSliceK rows of W_router (so the weight
// stream is spread over many SMs), write partial logits for all T tokens,
// and the last CTA to finish -- found with an atomic ticket after a memory
// fence, no waiting -- adds the partials in slice order (deterministic),
// adds the bias and does the rest alone.  It resets the ticket for the next
// launch.
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
constexpr int kSmallSliceK = 128;    // W_router rows per CTA
constexpr int kSmallThreads = 256;
constexpr int kSmallMaxEntries = kSmallMaxTokens * kMaxTopK;

// Dynamic shared memory: the x slice [T][kSmallSliceK] fp32 and the
// W_router slice [kSmallSliceK][E] in its storage type (both loaded with
// 16-byte vectors by every thread at once: one memory round trip), then the
// logits [T][E] fp32 (last CTA only, aliasing them).
template <typename ET>
__host__ __device__ constexpr size_t route_small_smem_bytes(int T, int E) {
    const size_t a = sizeof(float) * (size_t)T * kSmallSliceK + sizeof(ET) * (size_t)kSmallSliceK * E;
    const size_t b = sizeof(float) * (size_t)T * (size_t)E;
    return a > b ? a : b;
}

// Grid: ceil(d / kSmallSliceK) CTAs of kSmallThreads.  partial: [grid][T][E]
// fp32.  ticket: a word that is 0 when the launch starts (the finishing CTA
// leaves it at 0).  GT: the GEMMs' activation type (the layer's, f16 for
// 8-bit weights, or uint8_t E4M3 codes in the FP8 activation mode; x16 then
// receives x converted, token order, each row divided by its scale -- the
// power-of-two f16 range scale or the E4M3 row scale -- recorded in
// tokscale and folded into gslot).
template <typename ET, typename GT>
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(
    const ET* __restrict__ x, const ET* __restrict__ Wr, const float* __restrict__ bias, int T, int d,
    int E, int k, float* __restrict__ partial, unsigned* ticket, int32_t* __restrict__ idx,
    float* __restrict__ gate, float* __restrict__ lmax, float* __restrict__ margin,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
    int32_t* __restrict__ inv, float* __restrict__ gslot, GroupTable* tab_gu, GroupTable* tab_dn,
    int fb_gu_routed, int fb_gu_shared, int fb_down, GT* __restrict__ xg, GT* __restrict__ x16,
    float* __restrict__ tokscale) {
    pdl_enter();
    extern __shared__ float rs_smem[];
    __shared__ int32_t s_ent[kSmallMaxEntries];   // selected expert of entry n = t * k + j
    __shared__ int32_t s_rank[kSmallMaxEntries];  // rank of the entry inside its expert
    __shared__ float s_gate[kSmallMaxEntries];
    __shared__ int32_t s_rows[kMaxGroups];        // entries per expert
    __shared__ int32_t s_off[kMaxGroups + 1];     // exclusive prefix of s_rows
    __shared__ float s_scale[kSmallMaxTokens];    // row scale (converted rows; else 1)
    __shared__ unsigned s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---------------------------------------------- partial logits, one K slice
    {
        const int k0 = blockIdx.x * kSmallSliceK;
        const int kn = min(kSmallSliceK, d - k0);
        float* xs = rs_smem;                                                   // [T][kSmallSliceK]
        ET* ws = reinterpret_cast<ET*>(rs_smem + (size_t)T * kSmallSliceK);  // [kn][E]
        // the slice's rows of W_router are contiguous (kn * E elements): 16-byte
        // vectors, every thread at once, then the x slice (16-byte vectors too)
        {
            const int V = 16 / (int)sizeof(ET);
            const int nw = kn * E;  // E * sizeof(ET) need not be a multiple of 16: copy the flat range
            const ET* src = Wr + (size_t)k0 * E;
            const bool vec = ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) && (nw % V == 0);
            // each thread's loads of a pass are issued before any store (one
            // memory round trip per pass, not per vector)
            if (vec) {
                const int nv16 = nw / V;
                for (int i0 = tid; i0 < nv16; i0 += 8 * kSmallThreads) {
                    uint4 v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (i0 + j * kSmallThreads < nv16)
                            v[j] = reinterpret_cast<const uint4*>(src)[i0 + j * kSmallThreads];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (i0 + j * kSmallThreads < nv16) reinterpret_cast<uint4*>(ws)[i0 + j * kSmallThreads] = v[j];
                }
            } else {
                for (int i = tid; i < nw; i += kSmallThreads) ws[i] = src[i];
            }
            const int xv = kn / V;  // x rows: kn elements from k0 (k0, kn multiples of 64)
            const int nxv = T * xv;
            for (int i0 = tid; i0 < nxv; i0 += 4 * kSmallThreads) {
                uint4 raw[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j * kSmallThreads;
                    if (i < nxv) {
                        const int t = i / xv, c = i - t * xv;
                        raw[j] = reinterpret_cast<const uint4*>(x + (size_t)t * d + k0)[c];
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + j * kSmallThreads;
                    if (i >= nxv) continue;
                    const int t = i / xv, c = i - t * xv;
                    ET tmp[16 / sizeof(ET)];
                    *reinterpret_cast<uint4*>(tmp) = raw[j];
#pragma unroll
                    for (int u = 0; u < V; ++u) xs[t * kSmallSliceK + c * V + u] = to_f32(tmp[u]);
                }
            }
        }
        __syncthreads();
        // thread -> (expert e, token group g); a group takes tokens g, g + G,
        // ... (jn of them).  The loop bounds are held in registers (in_reg):
        // a kernel parameter read in the loop costs a constant-bank access
        // per use.
        const int nT = in_reg(T), nE = in_reg(E), nkn = in_reg(kn);
        const int G = max(1, kSmallThreads / nE);
        const int e = tid % nE, g = tid / nE;
        if (g < G && tid < G * nE) {
            const int jn = g < nT ? (nT - g + G - 1) / G : 0;  // tokens g + j * G < T
            float acc[kSmallMaxTokens];
#pragma unroll
            for (int j = 0; j < kSmallMaxTokens; ++j) acc[j] = 0.f;
            const ET* wcol = ws + e;
            const float* xg0 = xs + (size_t)g * kSmallSliceK;
            const int xstep = G * kSmallSliceK;
#pragma unroll 4
            for (int kk = 0; kk < nkn; ++kk) {
                const float w = to_f32(wcol[kk * nE]);
#pragma unroll
                for (int j = 0; j < kSmallMaxTokens; ++j)
                    if (j < jn) acc[j] = fmaf(xg0[j * xstep + kk], w, acc[j]);
            }
            float* p = partial + (size_t)blockIdx.x * nT * nE;
#pragma unroll
            for (int j = 0; j < kSmallMaxTokens; ++j)
                if (j < jn) p[(size_t)(g + j * G) * nE + e] = acc[j];
        }
    }
    // the last CTA to get here finishes the routing
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // ---------------------------------------------- logits: slices in order, + bias
    // each pass covers up to 4 outputs per thread (i = i0 + 256 q); the loads
    // of 8 slices for all of them are issued before any is added (one memory
    // round trip per 8 slices; 16 when a thread has one output), and each
    // output adds its slices in order
    float* lg = rs_smem;  // [T][E]
    const int nT = in_reg(T), nE = in_reg(E), nk = in_reg(k);
    {
        const int n = nT * nE;
        const int S = in_reg((int)gridDim.x);
        if (n <= kSmallThreads) {  // one output per thread: 16 slices per round trip
            if (tid < n) {
                float v = 0.f;
                for (int s0 = 0; s0 < S; s0 += 16) {
                    float ld[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u)
                        ld[u] = s0 + u < S ? __ldcg(partial + (size_t)(s0 + u) * n + tid) : 0.f;
#pragma unroll
                    for (int u = 0; u < 16; ++u)
                        if (s0 + u < S) v += ld[u];
                }
                lg[tid] = v + (bias ? bias[tid % nE] : 0.f);
            }
        }
        for (int i0 = tid; n > kSmallThreads && i0 < n; i0 += 4 * kSmallThreads) {
            float v[4] = {0.f, 0.f, 0.f, 0.f};
            for (int s0 = 0; s0 < S; s0 += 8) {
                float ld[8][4];
#pragma unroll
                for (int u = 0; u < 8; ++u)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i = i0 + kSmallThreads * q, sl = s0 + u;
                        ld[u][q] = (i < n && sl < S) ? __ldcg(partial + (size_t)sl * n + i) : 0.f;
                    }
#pragma unroll
                for (int u = 0; u < 8; ++u)
#pragma unroll
                    for (int q = 0; q < 4; ++q) v[q] += ld[u][q];
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = i0 + kSmallThreads * q;
                if (i < n) lg[i] = v[q] + (bias ? bias[i % nE] : 0.f);
            }
        }
    }
    __syncthreads();
    if (tid == 0) *ticket = 0u;  // every CTA has taken its ticket: ready for the next launch

    // ---------------------------------------------- top-k, one warp per token
    // each lane keeps the list of its experts (lane, lane + 32, ...: ascending,
    // so ties keep the lower index), then k + 1 butterfly rounds each take
    // the first head in (value, index) order
    for (int t = warp; t < nT; t += kSmallThreads / 32) {
        TopK tk;
        tk.init();
        for (int e = lane; e < nE; e += 32) tk.offer(lg[t * nE + e], e);
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
            sel.fill_empty(nk);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < nk) {
                    const int n = t * nk + j;
                    const float g = 1.0f / (1.0f + expf(-sel.value(j)));
                    idx[n] = sel.index(j);
                    lmax[n] = sel.value(j);
                    gate[n] = g;
                    s_ent[n] = sel.index(j);
                    s_gate[n] = g;
                }
            }
            margin[t] = sel.value(nk - 1) - sel.value(nk);
        }
    }
    for (int e = tid; e < nE; e += kSmallThreads) s_rows[e] = 0;
    // each token row's power-of-two scale into f16's range (8-bit weight
    // layers, f16_row_scale), one warp per token
    const int nv = in_reg(d * (int)sizeof(ET) / 16);
    for (int t = warp; t < nT; t += kSmallThreads / 32) {
        float sc = 1.0f;
        if constexpr (!std::is_same<ET, GT>::value) {
            float m = 0.0f;
            for (int i = lane; i < nv; i += 32) m = absmax_vec(reinterpret_cast<const uint4*>(x + (size_t)t * d)[i], m);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            sc = row_scale_of<ET, GT>(m);
            if (lane == 0 && tokscale) tokscale[t] = sc;
        }
        if (lane == 0) s_scale[t] = sc;
    }
    __syncthreads();

    // ---------------------------------------------- ranks, counts, offsets (warp 0)
    const int Tv = nT * nk;
    if (warp == 0) {
        for (int c0 = 0; c0 < Tv; c0 += 32) {
            const int n = c0 + lane;
            const int e = n < Tv ? s_ent[n] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int below = __popc(peers & ((1u << lane) - 1u));
            if (e >= 0) s_rank[n] = s_rows[e] + below;  // entries of e before this chunk, then this chunk's
            __syncwarp();
            if (e >= 0 && below == 0) s_rows[e] += __popc(peers);
            __syncwarp();
        }
        int local[8];
        int sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            local[j] = e < nE ? s_rows[e] : 0;
            sum += local[j];
        }
        const int incl = warp_incl_scan(sum);
        int acc = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            if (e < nE) {
                s_off[e] = acc;
                offsets[e] = acc;
                counts[e] = local[j];
            }
            acc += local[j];
        }
        if (lane == 31) {
            s_off[nE] = incl;
            offsets[nE] = incl;
        }
    }
    __syncthreads();
    for (int n = tid; n < Tv; n += kSmallThreads) {
        const int slot = s_off[s_ent[n]] + s_rank[n];
        inv[n] = slot;
        perm[slot] = n;
        gslot[slot] = s_gate[n] * s_scale[n / nk];
    }
    // candidate 0 is the shared expert, 1..E the routed experts
    build_tables(
        tab_gu, tab_dn, nE + 1, [&](int g) { return g == 0 ? nT : s_rows[g - 1]; },
        [&](int g) { return g == 0 ? 0 : s_off[g - 1]; }, [&](int g) { return g == 0 ? nE : g - 1; },
        [&](int g) { return g == 0 ? fb_gu_shared : fb_gu_routed; }, fb_down);

    // ---------------------------------------------- rows in expert order
    // xg[slot of n] = x[n / k] (16-byte vectors, converted for 8-bit weight
    // layers), and x16[t] = x[t] in token order when it is given
    const int rows = Tv + (x16 ? nT : 0);
    for (int i0 = tid; i0 < rows * nv; i0 += 4 * kSmallThreads) {
        uint4 raw[4];  // four 16-byte loads in flight before the stores
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kSmallThreads;
            if (i < rows * nv) {
                const int r = i / nv, c = i - r * nv;
                const int t = r >= Tv ? r - Tv : r / nk;
                raw[j] = reinterpret_cast<const uint4*>(x + (size_t)t * d)[c];
            }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = i0 + j * kSmallThreads;
            if (i >= rows * nv) continue;
            const int r = i / nv, c = i - r * nv;
            const bool tok = r >= Tv;
            const int t = tok ? r - Tv : r / nk;
            const int orow = tok ? t : s_off[s_ent[r]] + s_rank[r];
            put_row_vec<ET, GT>((tok ? x16 : xg) + (size_t)orow * d, c, raw[j], row_scale(s_scale[t]));
        }
    }
}

}  // namespace l4moe
