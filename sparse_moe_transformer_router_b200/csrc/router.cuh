// router.cuh -- router logits, top-1 selection and the sigmoid gate.
//
// superteams.ai "Llama 4" glossary, section "Mixture of Experts: Why Total
// and Active Parameters Diverge": the router scores every expert once per
// token and the token goes to the single best one.  KerasFormers "Llama 4",
// section "What is unusual about the block": the chosen expert is reached
// through a sigmoid gate on its input.
//
// One CTA handles TT = NT / TPT tokens; TPT threads share a token and each
// owns NG groups of 4 consecutive experts.  x and W_router are staged through
// shared memory in K chunks of 64 and converted to fp32; each thread keeps
// 4 * NG fp32 accumulators (sequential fma over k).  The per-token arg-max
// uses a strict ">" in ascending expert order inside a thread and "larger
// value, then lower index" across threads, which is the sequential rule
// "lowest index among the maxima; NaN never wins".
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

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
                                                    float* __restrict__ margin) {
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

    // thread-local best / runner-up in ascending expert order
    float best = -INFINITY, second = -INFINITY;
    int bi = (4 * r < E) ? 4 * r : 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NG; ++j) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int e = 4 * (r + TPT * j) + c;
            if (e < E) {
                const float l = acc[j][c] + (bias ? bias[e] : 0.f);
                if (l > best) {
                    second = best;
                    best = l;
                    bi = e;
                } else if (l > second) {
                    second = l;
                }
            }
        }
    }
    // combine the TPT threads of this token (consecutive lanes)
#pragma unroll
    for (int off = TPT / 2; off > 0; off /= 2) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const float os = __shfl_xor_sync(0xffffffffu, second, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ob > best || (ob == best && oi < bi)) {
            second = fmaxf(os, best);
            best = ob;
            bi = oi;
        } else {
            second = fmaxf(second, ob);
        }
    }
    const int t = t0 + tl;
    if (r == 0 && t < T) {
        idx[t] = bi;
        lmax[t] = best;
        margin[t] = best - second;
        gate[t] = 1.0f / (1.0f + expf(-best));
    }
}

}  // namespace l4moe
