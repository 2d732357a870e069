// quant.cuh -- E4M3 row quantisation of the FP8 activation mode.
//
// superteams.ai "Llama 4" glossary, "Running Llama 4 Yourself": Maverick is
// served with FP8 quantisation.  In this mode every contraction input row --
// a token's x, and each hidden row an expert produces -- is quantised to
// OCP E4M3 with one fp32 scale for the row:
//   s = fp32(max|v| / 448)  (1 for a row of zeros),
//   code = e4m3_rne_satfinite(fp32(v / s)),
// and the contraction reads code * s.  Both steps are IEEE fp32 operations
// (a correctly rounded division, not a multiply by 1 / s), so the codes are
// a function of the row alone.  The hidden rows are stored in bf16 first:
// the scale needs the maximum of the whole row, which spans many GEMM
// output tiles, so one kernel writes the row and the next quantises it.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace l4moe {

// The row scale from the row's largest magnitude.
__device__ __forceinline__ float e4m3_row_scale(float amax) {
    const float s = __fdiv_rn(amax, 448.0f);
    return s == 0.0f ? 1.0f : s;
}

// Two fp32 values -> two E4M3 codes (lo at the lower address), round to
// nearest even, finite values beyond 448 saturate to +-448.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// 8 bf16 values (16 bytes) divided by s -> 8 codes (8 bytes, element order).
__device__ __forceinline__ uint2 bf16x8_to_e4m3(uint4 v, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        c[i] = f32x2_to_e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
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
// shapes, one byte each) and scales sc_r [Tr] / sc_s [T].  One warp per row,
// 16-byte loads; the second pass re-reads the row from L1/L2.  F, Fs
// multiples of 8.
__global__ void __launch_bounds__(256) quant_hidden_kernel(const __nv_bfloat16* __restrict__ h_r,
                                                           const __nv_bfloat16* __restrict__ h_s, int Tr,
                                                           int T, int F, int Fs, uint8_t* __restrict__ q_r,
                                                           uint8_t* __restrict__ q_s, float* __restrict__ sc_r,
                                                           float* __restrict__ sc_s) {
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < Tr + T; r += warps) {
        const bool sh = r >= Tr;
        const int row = sh ? r - Tr : r;
        const int w = sh ? Fs : F;
        const uint4* src = reinterpret_cast<const uint4*>((sh ? h_s : h_r) + (size_t)row * w);
        uint2* dst = reinterpret_cast<uint2*>((sh ? q_s : q_r) + (size_t)row * w);
        const int nv = w / 8;
        float m = 0.0f;
        for (int i = lane; i < nv; i += 32) m = absmax_vec(src[i], m);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float s = e4m3_row_scale(m);
        if (lane == 0) (sh ? sc_s : sc_r)[row] = s;
        for (int i = lane; i < nv; i += 32) dst[i] = bf16x8_to_e4m3(src[i], s);
    }
}

}  // namespace l4moe
