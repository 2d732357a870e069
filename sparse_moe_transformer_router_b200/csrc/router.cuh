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

#include "permute.cuh"
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
// selected logit minus the next one): the CTAs of a 128-token tile compute
// the fp32 logits of all E experts with tcgen05 (M = 128 tokens, N = E
// rounded up to 16, K = d or a slice of it; x rows are the K-major A operand,
// W_router [d, E] the MN-major B operand), then the lanes that finish a
// token apply the same arg-max / runner-up / sigmoid rule as the CUDA-core
// router above (details at the kernel).  Warp 0 lane 0 issues the TMA loads,
// warp 1 lane 0 the MMAs; all four warps run the epilogue.
namespace rmma {
constexpr int A_BYTES = 128 * 128;     // 128 tokens x 64 K (bf16)
constexpr int B_BOX_BYTES = 64 * 128;  // 64 K rows x 64 experts (bf16)
constexpr int MAX_STAGES = 6;
// The largest dynamic shared memory a launch asks for (stages, barriers,
// slack), leaving room for the kernel's static shared memory.
constexpr size_t SMEM_BYTES = 224 * 1024;
// A launch whose CTAs each take n_chunk experts needs stages of the token
// tile plus ceil(n_chunk / 64) weight boxes only: fewer bytes, so that two
// CTAs fit on an SM when the experts are few.
__host__ __device__ constexpr int stage_bytes(int n_chunk) {
    return A_BYTES + ((n_chunk + 63) / 64) * B_BOX_BYTES;
}
__host__ __device__ constexpr size_t smem_bytes(int n_chunk, int nst) {
    return 1024 + (size_t)nst * stage_bytes(n_chunk) + (2 * nst + 1) * 8 + 16;
}
// Stages of a launch: 4 when two CTAs then share an SM (each at most half of
// its shared memory), else as many as one CTA's shared memory holds, up to
// MAX_STAGES -- the bytes in flight per SM are what keep the x stream at the
// HBM rate.
__host__ __device__ constexpr int stages(int n_chunk) {
    return smem_bytes(n_chunk, 4) <= 112 * 1024 ? 4
           : (int)((SMEM_BYTES - 1024 - 16 - 8) / (stage_bytes(n_chunk) + 16)) < MAX_STAGES
               ? (int)((SMEM_BYTES - 1024 - 16 - 8) / (stage_bytes(n_chunk) + 16))
               : MAX_STAGES;
}
}  // namespace rmma

// The dispatch a top-1 router launch may finish itself (chunk_base not
// null): the tokens each CTA finishes (tokens_per_cta of one 128-token tile,
// below) form a dispatch chunk whose stable ranks go to inv[t] and whose
// per-expert counts go to chunk_base[chunk][E]; the last CTA to finish
// (atomic ticket after a memory fence, no waiting) writes the chunk bases,
// counts, offsets and the two work lists (dispatch_finish) and resets the
// ticket.  The outputs are those of dispatch_kernel with chunks of
// tokens_per_cta entries.
struct RouterDispatch {
    int32_t* chunk_base;  // [chunks][E]
    int32_t* counts;      // [E]
    int32_t* offsets;     // [E + 1]
    int32_t* inv;         // [T]: rank inside (chunk, expert)
    GroupTable* tab_gu;
    GroupTable* tab_dn;
    unsigned* ticket;     // zero between launches
    int fb_gu_routed, fb_gu_shared, fb_down;
};

// Tokens of a tile that each CTA of a K-split launch (S slices) finishes.
__host__ __device__ constexpr int router_tokens_per_cta(int S) { return 128 / S; }

// Ints of a dispatching router CTA's stage memory left for the staging of
// the last CTA's scan (after tot and soff); the launch dispatches only when
// its chunks fit (a row of E per chunk, or at least one column).
__host__ __device__ constexpr int router_stage_cap(int E) {
    return (int)((size_t)rmma::stages(E) * rmma::stage_bytes(E) / 4) - ((2 * E + 1 + 3) & ~3);
}

// A kernel parameter copied into a register the compiler cannot re-derive:
// the epilogue's loops otherwise re-read such scalars from the constant
// bank on every element, which costs tens of cycles each.
__device__ __forceinline__ int in_reg(int v) {
    int r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
    return r;
}

__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// 16 bytes to a shared::cluster address (this or another CTA of the cluster).
__device__ __forceinline__ void st_shared_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}
// 16 bytes to this CTA's shared memory.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// K split (gridDim.z = S slices, S a power of two <= 8, launched as clusters
// of (1, 1, S) when S > 1): CTA z of a cluster computes the partial logits
// of the same 128 tokens over K slice z.  The slices then meet in the CTA
// that finishes each token: CTA z owns the tile's tokens [z * 128 / S,
// (z + 1) * 128 / S).  After a cluster barrier (every CTA's operand stages
// are idle), each thread stores its token row's partial (TMEM lane = token)
// into the owner's shared memory, slot z: recv[S][128 / S][n_pad + 4] fp32;
// a second barrier (release / acquire) makes the rows visible.  The owner's
// S consecutive lanes per token each sum a 1/S share of the experts over the
// slices in order 0 .. S-1 (deterministic), then merge their arg-max (or
// top-k) with shuffles.  With S = 1 the same exchange runs inside the CTA.
// This spreads the x stream of a batch of few token tiles over S times more
// SMs and keeps the reduction parallel: no CTA waits on remote loads.
//
// Expert-split mode (logits != null, for batches of one token tile): CTA
// (y, z) computes experts [y*n_chunk, (y+1)*n_chunk) over K slice z of
// gridDim.z; the slices meet as above and the owners store the biased fp32
// logits to logits[T][E]; the arg-max then runs in the permutation kernel.
// This spreads the router weight stream over (E / n_chunk) x slices SMs
// instead of one.
__global__ void __launch_bounds__(128, 2)
    router_mma_kernel(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap wr_map,
                      const float* __restrict__ bias, int T, int d, int E, int n_chunk,
                      float* __restrict__ logits, int32_t* __restrict__ idx,
                      float* __restrict__ gate, float* __restrict__ lmax,
                      float* __restrict__ margin, unsigned* err, int topk, int nst, const RouterDispatch dsp) {
    extern __shared__ uint8_t rsmem_raw[];
    __shared__ unsigned s_last;
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(rsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int stage_bytes = rmma::stage_bytes(n_chunk);  // this launch's stage stride
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)nst * stage_bytes);  // nst stages
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * nst + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t stage0 = smem_u32(smem), bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (nst + s); };
    const uint32_t done_bar = bar0 + 8u * (2 * nst);
    const int e0 = blockIdx.y * n_chunk;        // first expert of this CTA
    const int ne = min(n_chunk, E - e0);         // experts of this CTA
    const int n_pad = (ne + 15) & ~15;
    const int nbb = (ne + 63) / 64;
    uint32_t ncols = 32;
    while ((int)ncols < n_pad) ncols <<= 1;

    // set-up that touches no input: before the wait on the preceding kernel
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(done_bar, 1);
        fence_barrier_init();
        tma_prefetch_desc(&x_map);
        tma_prefetch_desc(&wr_map);
    }
    pdl_enter();
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
            if (++stage == nst) {
                stage = 0;
                phase ^= 1u;
            }
        }
        for (int s = 0; s < nst; ++s)  // drain copies in flight
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
            if (++stage == nst) {
                stage = 0;
                phase ^= 1u;
            }
        }
        mma_commit(done_bar);  // logits complete (or every issued MMA finished)
    }
    __syncwarp();
    const bool ok = mbar_wait(done_bar, 0, err, DEV_ERR_TIMEOUT_EPILOGUE);
    const bool all_ok = __syncthreads_and(ok) != 0;  // CTA-uniform from here on

    // ---- the slices meet in the CTA that owns each token (see above)
    const int S = in_reg((int)gridDim.z);
    const uint32_t z = S > 1 ? cluster_ctarank() : 0u;
    const int tpc = router_tokens_per_cta(S);
    const int rld = n_pad + 4;                           // recv row stride (floats)
    float* recv = reinterpret_cast<float*>(smem);        // [S][tpc][rld] in the idle stages
    const int row = 32 * warp + lane;                    // this thread's token row (TMEM lane)
    const uint32_t dst_local = smem_u32(recv + ((size_t)z * tpc + row % tpc) * rld);
    if (S > 1) cluster_arrive_release();  // this CTA's stages are idle: the others may write them
    const uint32_t dst = S > 1 ? mapa_shared(dst_local, (uint32_t)(row / tpc)) : dst_local;
    if (S > 1) cluster_wait_acquire();
    if (all_ok) {
        tc_fence_after();
        for (int c = 0; c < n_pad; c += 32) {
            float v[32];
            tmem_ld_32x32(tmem_base + ((uint32_t)(32 * warp) << 16) + (uint32_t)c, v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (c + 4 * q >= n_pad) continue;
                const uint32_t a = dst + 4u * (uint32_t)(c + 4 * q);
                if (S > 1) st_shared_cluster_v4(a, v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                else st_shared_v4(a, v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
    }
    if (S > 1) {
        cluster_arrive_release();  // every row stored ...
        cluster_wait_acquire();    // ... and visible to its owner
    } else {
        __syncthreads();
    }

    // ---- this CTA's tokens: S consecutive lanes per token, lane `sub` takes
    // experts [sub * ne / S, (sub + 1) * ne / S) of the CTA's ne (S divides ne)
    const int nE = in_reg(E), nT = in_reg(T), nK = in_reg(topk);
    const bool has_bias = bias != nullptr;
    const int rl = threadIdx.x / S, sub = threadIdx.x - rl * S;
    const int t = t0 + (int)z * tpc + rl;
    const int per = in_reg(ne / S);
    const int eb = sub * per;
    const int rld_r = in_reg(rld);
    const float* rrow = recv + (size_t)rl * rld_r;           // slot 0 of this token's rows
    const size_t slot_stride = (size_t)tpc * rld_r;
    auto logit = [&](int e) {  // sum over the slices in order, then the bias
        float p[8];
#pragma unroll
        for (int s = 0; s < 8; ++s) p[s] = s < S ? rrow[s * slot_stride + e] : 0.f;  // loads first
        float l = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s)
            if (s < S) l += p[s];
        return has_bias ? l + bias[e0 + e] : l;
    };
    int e_tok = -1;  // top-1: the token's expert in its lane sub == 0 (-1 past T or on failure)
    if (all_ok) {
        if (logits) {
            for (int e = eb; e < eb + per; ++e)
                if (t < nT) logits[(size_t)t * nE + e0 + e] = logit(e);
        } else if (nK == 1) {
            // this lane's share: the arg-max (strict ">" in ascending order:
            // the lowest index among the maxima; NaN never wins) and the
            // runner-up, branch-free
            float best = -INFINITY, second = -INFINITY;
            int bi = eb;
            auto offer = [&](float l, int e) {
                const bool gt = l > best;
                second = gt ? best : fmaxf(second, l);
                bi = gt ? e : bi;
                best = gt ? l : best;
            };
            if ((per & 3) == 0) {  // four experts per step: 16-byte loads of every slice first
                for (int e = eb; e < eb + per; e += 4) {
                    float4 p[8];
#pragma unroll
                    for (int s = 0; s < 8; ++s)
                        p[s] = s < S ? *reinterpret_cast<const float4*>(rrow + s * slot_stride + e)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                    float4 l = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        if (s >= S) continue;
                        l.x += p[s].x;
                        l.y += p[s].y;
                        l.z += p[s].z;
                        l.w += p[s].w;
                    }
                    if (has_bias) {
                        l.x += bias[e0 + e];
                        l.y += bias[e0 + e + 1];
                        l.z += bias[e0 + e + 2];
                        l.w += bias[e0 + e + 3];
                    }
                    offer(l.x, e);
                    offer(l.y, e + 1);
                    offer(l.z, e + 2);
                    offer(l.w, e + 3);
                }
            } else {
#pragma unroll 4
                for (int e = eb; e < eb + per; ++e) offer(logit(e), e);
            }
            // merge the token's S shares: larger value first, then lower index
            for (int off = S >> 1; off > 0; off >>= 1) {
                const float ob = __shfl_xor_sync(0xffffffffu, best, off);
                const float os = __shfl_xor_sync(0xffffffffu, second, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                const bool take = ob > best || (ob == best && oi < bi);
                second = fmaxf(fmaxf(second, os), take ? best : ob);
                bi = take ? oi : bi;
                best = take ? ob : best;
            }
            if (sub == 0 && t < nT) {
                idx[t] = bi;
                lmax[t] = best;
                gate[t] = 1.0f / (1.0f + expf(-best));
                margin[t] = best - second;
                e_tok = bi;
            }
        } else {
            TopK tk;
            tk.init();
            for (int e = eb; e < eb + per; ++e) tk.offer(logit(e), e);
            // the token's S lists (consecutive lanes): k + 1 heads in selection order
            TopK sel;
            sel.init();
            int pos = 0;  // entries of this lane's list already taken
#pragma unroll
            for (int j = 0; j <= kMaxTopK; ++j) {
                float hv = tk.value(pos);
                int hi = pos <= kMaxTopK ? tk.index(pos) : -1;
                int hl = sub;
                for (int off = S >> 1; off > 0; off >>= 1) {
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
                if (hl == sub && hi >= 0) ++pos;
            }
            if (sub == 0 && t < nT) {
                sel.fill_empty(nK);
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j) {
                    if (j < nK) {
                        const size_t n = (size_t)t * nK + j;
                        idx[n] = sel.index(j);
                        lmax[n] = sel.value(j);
                        gate[n] = 1.0f / (1.0f + expf(-sel.value(j)));
                    }
                }
                margin[t] = sel.value(nK - 1) - sel.value(nK);  // k-th against the next one
            }
        }
    }

    if (dsp.chunk_base) {
        // this CTA's tokens are one dispatch chunk; the ranks' counts follow
        // recv, and the last CTA's scan reuses the whole stage memory (recv
        // and wcnt are idle by then)
        int* wcnt = reinterpret_cast<int*>(recv + (size_t)S * slot_stride);  // [4][E]
        int* tot = reinterpret_cast<int*>(smem);
        int* soff = tot + nE;
        int* stage = tot + ((2 * nE + 1 + 3) & ~3);  // 16-byte aligned
        const int chunk = blockIdx.x * S + (int)z;
        const int r = chunk_rank(e_tok, nE, wcnt, dsp.chunk_base + (size_t)chunk * nE);
        if (sub == 0 && t < nT) dsp.inv[t] = r;
        __threadfence();
        __syncthreads();
        const unsigned ctas = gridDim.x * (unsigned)S;
        if (threadIdx.x == 0) s_last = (atomicAdd(dsp.ticket, 1u) == ctas - 1u) ? 1u : 0u;
        __syncthreads();
        if (s_last) {
            __threadfence();
            const int cap = router_stage_cap(nE);  // >= the chunks (the host dispatches here only then)
            dispatch_finish<8>(dsp.chunk_base, (int)ctas, nT, nE, dsp.fb_gu_routed, dsp.fb_gu_shared, dsp.fb_down,
                               dsp.counts, dsp.offsets, dsp.tab_gu, dsp.tab_dn, tot, soff, stage, cap);
            if (threadIdx.x == 0) *dsp.ticket = 0u;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, ncols);
    }
}

}  // namespace l4moe
