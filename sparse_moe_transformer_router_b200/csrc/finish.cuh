// finish.cuh -- the kernels that close a GEMM launch made of fp32 partials:
// the split-K sum of the gate/up contraction (with the gate and SwiGLU), and
// the down projection's sum of the routed and shared partials, rounded once.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <type_traits>

#include "moe_gemm.cuh"
#include "ptx.cuh"

namespace l4moe {

// Split-K finish of the gate/up contraction: h = silu(g * sum_s a_gate) *
// (g * sum_s a_up) over the splits in order, for the routed slots (g = the
// slot's sigmoid gate, times its row's power-of-two scale for 8-bit weight
// layers) and the shared rows (g = 1, or the token's row scale: tokscale).
// One thread per output.
template <typename ET>
__global__ void __launch_bounds__(256) gateup_finish_kernel(
    const float* __restrict__ part_r, long long ld_r, long long stride_r, const float* __restrict__ part_s,
    long long ld_s, long long stride_s, int ksplit, int Tr, int T, int F, int Fs,
    const float* __restrict__ gslot, const float* __restrict__ tokscale, ET* __restrict__ hr,
    ET* __restrict__ hs, unsigned* err) {
    pdl_enter();
    // Tr routed rows (token entries), T shared rows
    const long long n_r = (long long)Tr * F, n = n_r + (long long)T * Fs;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const bool shared = i >= n_r;
        const long long j = shared ? i - n_r : i;
        const int w = shared ? Fs : F;
        const int row = (int)(j / w), f = (int)(j % w);
        const float* p = shared ? part_s : part_r;
        const long long ld = shared ? ld_s : ld_r, st = shared ? stride_s : stride_r;
        float ag = 0.f, au = 0.f;
        for (int s = 0; s < ksplit; ++s) {
            ag += p[st * s + (long long)row * ld + f];
            au += p[st * s + (long long)row * ld + w + f];
        }
        const float g = shared ? (tokscale ? tokscale[row] : 1.0f) : gslot[row];
        const float hv = silu_f(g * ag) * (g * au);
        if (sizeof(ET) == 2 && !std::is_same<ET, __nv_bfloat16>::value && !(fabsf(hv) < 65520.0f))
            atomicOr(err, DEV_ERR_F16_RANGE);  // f16 hidden rows (8-bit weights): out of range
        store_elem((shared ? hs : hr) + (long long)row * w + f, hv);
    }
}

// Four fp32 sums -> outputs 4i .. 4i+3, rounded once to the output type.
template <typename ET>
__device__ __forceinline__ void store_out4(ET* out, long long i, float4 acc) {
    if constexpr (sizeof(ET) == 2) {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi);
        reinterpret_cast<uint2*>(out)[i] = pk;
    } else {
        reinterpret_cast<float4*>(out)[i] = acc;
    }
}

// Down finish: out[t] = rn(sum over splits s and selected experts j of the
// routed partial of entry t * k + j, then sum over s of the shared partial)
// -- one rounding, a fixed order.  Partials: routed [splits_r][T * k][d],
// shared [splits_s][T][d] (fp32, rows un-permuted to entries / tokens).
// Four outputs per thread; d % 4 == 0.  done (fused launches, else null):
// the fused GEMM's two tile counters, reset here for the next forward (the
// GEMM has finished: this kernel's entry waits for it).
template <typename ET>
__global__ void __launch_bounds__(256) down_finish_kernel(const float* __restrict__ part_r, long long stride_r,
                                                          int splits_r, const float* __restrict__ part_s,
                                                          long long stride_s, int splits_s, int k, int d,
                                                          long long n, ET* __restrict__ out, unsigned* done) {
    pdl_enter();
    if (done && blockIdx.x == 0 && threadIdx.x < 2) done[threadIdx.x] = 0u;
    const long long n4 = n >> 2;
    const int d4 = d >> 2;
    const long long stride = (long long)gridDim.x * blockDim.x;
    long long i0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (k == 1 && splits_r == 1 && splits_s == 1) {
        // one routed and one shared partial per output (prefill): two outputs
        // per thread and pass, their four loads issued before any is used,
        // so that enough bytes are in flight to keep HBM busy
        for (; i0 < n4; i0 += 2 * stride) {
            const long long i1 = i0 + stride;
            const bool two = i1 < n4;
            const float4 r0 = reinterpret_cast<const float4*>(part_r)[i0];
            const float4 s0 = reinterpret_cast<const float4*>(part_s)[i0];
            float4 r1 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = r1;
            if (two) {
                r1 = reinterpret_cast<const float4*>(part_r)[i1];
                s1 = reinterpret_cast<const float4*>(part_s)[i1];
            }
            store_out4(out, i0, make_float4(r0.x + s0.x, r0.y + s0.y, r0.z + s0.z, r0.w + s0.w));
            if (two) store_out4(out, i1, make_float4(r1.x + s1.x, r1.y + s1.y, r1.z + s1.z, r1.w + s1.w));
        }
        return;
    }
    for (long long i = i0; i < n4; i += stride) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k == 1) {  // routed row t is entry t: the same index as the output
            // the partials of up to 8 splits are loaded before any is added
            // (a small batch is latency-bound here: one round trip per 8)
            for (int s0 = 0; s0 < splits_r; s0 += 8) {
                float4 v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    v[j] = s0 + j < splits_r ? reinterpret_cast<const float4*>(part_r + stride_r * (s0 + j))[i]
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < 8; ++j) acc.x += v[j].x, acc.y += v[j].y, acc.z += v[j].z, acc.w += v[j].w;
            }
        } else {
            const long long t = i / d4, c4 = i - t * d4;
            for (int s = 0; s < splits_r; ++s)
                for (int j = 0; j < k; ++j) {
                    const float4 v =
                        reinterpret_cast<const float4*>(part_r + stride_r * s)[(t * k + j) * d4 + c4];
                    acc.x += v.x, acc.y += v.y, acc.z += v.z, acc.w += v.w;
                }
        }
        for (int s0 = 0; s0 < splits_s; s0 += 8) {
            float4 v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                v[j] = s0 + j < splits_s ? reinterpret_cast<const float4*>(part_s + stride_s * (s0 + j))[i]
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc.x += v[j].x, acc.y += v[j].y, acc.z += v[j].z, acc.w += v[j].w;
        }
        store_out4(out, i, acc);
    }
}

}  // namespace l4moe
