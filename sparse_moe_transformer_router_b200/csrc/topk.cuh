// topk.cuh -- the selected experts of one token: the k largest router logits
// (k <= kMaxTopK), in descending order, the lower index first among equal
// values, NaN never selected.  With k = 1 this is the arg-max of the
// superteams.ai "Llama 4" glossary's routing sketch; k > 1 is the "experts
// per token" choice of a token-choice router (torchtune MoE documentation).
#pragma once
#include <cstdint>
#include <cmath>

namespace l4moe {

constexpr int kMaxTopK = 4;

// The kMaxTopK + 1 largest values offered so far, descending; offers come in
// ascending expert order, so a strict ">" keeps an equal value behind the
// earlier (lower) index.  Empty slots (index -1) sit at the end and take any
// non-NaN value, -inf included; NaN is never taken.  The slots are separate
// scalars, not an array, so that the list lives in registers whatever the
// compiler decides about unrolling the loops around it.
struct TopK {
    float v0, v1, v2, v3, v4;
    int i0, i1, i2, i3, i4;

    __host__ __device__ __forceinline__ void init() {
        v0 = v1 = v2 = v3 = v4 = -INFINITY;
        i0 = i1 = i2 = i3 = i4 = -1;
    }
    __host__ __device__ __forceinline__ static bool beats(float l, float v, int i) {
        return l > v || (i < 0 && l == l);
    }
    // Insert from the bottom: each slot that l beats moves down one place.
    __host__ __device__ __forceinline__ void offer(float l, int e) {
        if (!beats(l, v4, i4)) return;
        if (!beats(l, v3, i3)) { v4 = l; i4 = e; return; }
        v4 = v3; i4 = i3;
        if (!beats(l, v2, i2)) { v3 = l; i3 = e; return; }
        v3 = v2; i3 = i2;
        if (!beats(l, v1, i1)) { v2 = l; i2 = e; return; }
        v2 = v1; i2 = i1;
        if (!beats(l, v0, i0)) { v1 = l; i1 = e; return; }
        v1 = v0; i1 = i0;
        v0 = l; i0 = e;
    }
    // Slot j (0 .. kMaxTopK; larger j reads the last slot).
    __host__ __device__ __forceinline__ float value(int j) const {
        return j <= 0 ? v0 : j == 1 ? v1 : j == 2 ? v2 : j == 3 ? v3 : v4;
    }
    __host__ __device__ __forceinline__ int index(int j) const {
        return j <= 0 ? i0 : j == 1 ? i1 : j == 2 ? i2 : j == 3 ? i3 : i4;
    }
    __host__ __device__ __forceinline__ void set(int j, float v, int i) {
        if (j == 0) { v0 = v; i0 = i; }
        else if (j == 1) { v1 = v; i1 = i; }
        else if (j == 2) { v2 = v; i2 = i; }
        else if (j == 3) { v3 = v; i3 = i; }
        else { v4 = v; i4 = i; }
    }
    // Slots left empty (only NaN logits were left) take the lowest indices
    // not selected yet, as a sequential scan would.
    __host__ __device__ __forceinline__ void fill_empty(int k) {
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k && index(j) < 0) {
                int e = 0;
                bool clash = true;
                while (clash) {
                    clash = false;
#pragma unroll
                    for (int q = 0; q < kMaxTopK; ++q)
                        if (q < j && index(q) == e) clash = true;
                    if (clash) ++e;
                }
                set(j, value(j), e);
            }
        }
    }
};

// "a before b" in the selection order: non-empty before empty, larger value,
// then lower index.
__host__ __device__ __forceinline__ bool topk_before(float av, int ai, float bv, int bi) {
    if (ai < 0) return false;
    if (bi < 0) return true;
    return av > bv || (av == bv && ai < bi);
}

}  // namespace l4moe
