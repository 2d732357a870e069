// quant.cuh -- E4M3 row quantisation of the FP8 activation mode.
//
// superteams.ai "Llama 4" glossary, "Running Llama 4 Yourself": Maverick is
// served with FP8 quantisation.  In this mode every contraction input row --
// a token's x, and each hidden row an expert produces -- is quantised to
// OCP E4M3 with one fp32 scale for the row:
//   s = fp32(max|v| / 448), at least 2^-126 (so that 1 / s is finite), and
//       1 for a row of zeros,
//   code = e4m3_rne_satfinite(fp32(v * fp32(1 / s))),
// and the contraction reads code * s.  Every step is an IEEE fp32 operation
// (a correctly rounded division for s and for 1 / s, one rounded product per
// value), so the codes are a function of the row alone.  The hidden rows are
// stored in bf16 first: the scale needs the maximum of the whole row, which
// spans many GEMM output tiles, so one kernel writes the row and the next
// quantises it.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace l4moe {

// The row scale from the row's largest magnitude.
__device__ __forceinline__ float e4m3_row_scale(float amax) {
    if (amax == 0.0f) return 1.0f;
    return fmaxf(__fdiv_rn(amax, 448.0f), 0x1p-126f);
}

// Two fp32 values -> two E4M3 codes (lo at the lower address), round to
// nearest even, finite values beyond 448 saturate to +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// A row's scale s and its correctly rounded reciprocal r (also the exact
// reciprocal of the power-of-two f16 range scales of 8-bit weight layers).
struct RowScale {
    float s, r;
};

__device__ __forceinline__ RowScale row_scale(float s) {
    RowScale q;
    q.s = s;
    q.r = __frcp_rn(s);
    return q;
}

// 8 bf16 values (16 bytes) times the row's reciprocal scale -> 8 codes (8
// bytes, element order).
__device__ __forceinline__ uint2 bf16x8_to_e4m3(uint4 v, const RowScale& q) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        c[i] = f32x2_to_e4m3x2(__fmul_rn(f.x, q.r), __fmul_rn(f.y, q.r));
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// Largest |x| of 8 bf16 values.
__device__ __forceinline__ float absmax_vec(uint4 v, float m) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return m;
}

// Hidden rows -> E4M3 codes and row scales: the routed rows h_r [Tr][F] and
// the shared rows h_s [T][Fs] (bf16, row-major) become codes q_r / q_s (same
// shapes, one byte each) and scales sc_r [Tr] / sc_s [T].  One CTA of
// kQuantThreads per row at a time: each thread loads up to kQuantVecs
// 16-byte vectors of the row into registers (rows of up to 16384 features;
// wider rows read the rest twice), the CTA reduces the row's largest magnitude,
// and the same registers are quantised and stored -- one read of the row
// from DRAM.  F, Fs multiples of 8.
constexpr int kQuantThreads = 256;
constexpr int kQuantVecs = 8;

__global__ void __launch_bounds__(kQuantThreads) quant_hidden_kernel(
    const __nv_bfloat16* __restrict__ h_r, const __nv_bfloat16* __restrict__ h_s, int Tr, int T, int F, int Fs,
    uint8_t* __restrict__ q_r, uint8_t* __restrict__ q_s, float* __restrict__ sc_r, float* __restrict__ sc_s) {
    pdl_enter();
    __shared__ float red[kQuantThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int r = blockIdx.x; r < Tr + T; r += gridDim.x) {
        const bool sh = r >= Tr;
        const int row = sh ? r - Tr : r;
        const int w = sh ? Fs : F;
        const uint4* src = reinterpret_cast<const uint4*>((sh ? h_s : h_r) + (size_t)row * w);
        uint2* dst = reinterpret_cast<uint2*>((sh ? q_s : q_r) + (size_t)row * w);
        const int nv = w / 8;
        uint4 v[kQuantVecs];
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < kQuantVecs; ++j) {
            const int i = tid + kQuantThreads * j;
            v[j] = i < nv ? __ldcs(src + i) : make_uint4(0u, 0u, 0u, 0u);
            m = absmax_vec(v[j], m);
        }
        for (int i = tid + kQuantThreads * kQuantVecs; i < nv; i += kQuantThreads) m = absmax_vec(src[i], m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) red[warp] = m;
        __syncthreads();
        m = red[0];
#pragma unroll
        for (int i = 1; i < kQuantThreads / 32; ++i) m = fmaxf(m, red[i]);
        const RowScale q = row_scale(e4m3_row_scale(m));
        if (tid == 0) (sh ? sc_s : sc_r)[row] = q.s;
#pragma unroll
        for (int j = 0; j < kQuantVecs; ++j) {
            const int i = tid + kQuantThreads * j;
            if (i < nv) dst[i] = bf16x8_to_e4m3(v[j], q);
        }
        for (int i = tid + kQuantThreads * kQuantVecs; i < nv; i += kQuantThreads) dst[i] = bf16x8_to_e4m3(src[i], q);
        __syncthreads();  // red[] is rewritten for the next row
    }
}

}  // namespace l4moe
