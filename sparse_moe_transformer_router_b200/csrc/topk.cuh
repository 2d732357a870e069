// topk.cuh -- the selected experts of one token: the k largest router logits
// (k <= kMaxTopK), in descending order, the lower index first among equal
// values, NaN never selected.  With k = 1 this is the arg-max of the
// superteams.ai "Llama 4" glossary's routing sketch; k > 1 is the "experts
// per token" choice of a token-choice router (torchtune MoE documentation).
#pragma once
#include <cstdint>

namespace l4moe {

constexpr int kMaxTopK = 4;

// The kMaxTopK + 1 largest values offered so far, descending; offers come in
// ascending expert order, so a strict ">" keeps an equal value behind the
// earlier (lower) index.  Empty slots (index -1) sit at the end and take any
// non-NaN value, -inf included; NaN is never taken.  All indexing is
// compile-time, so the list stays in registers.
struct TopK {
    float v[kMaxTopK + 1];
    int i[kMaxTopK + 1];

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int j = 0; j <= kMaxTopK; ++j) {
            v[j] = -INFINITY;
            i[j] = -1;
        }
    }
    __device__ __forceinline__ bool beats(float l, int j) const {
        return l > v[j] || (i[j] < 0 && l == l);
    }
    __device__ __forceinline__ void offer(float l, int e) {
        if (!beats(l, kMaxTopK)) return;
#pragma unroll
        for (int j = kMaxTopK; j > 0; --j) {
            if (beats(l, j - 1)) {  // slot j - 1 moves down one place
                v[j] = v[j - 1];
                i[j] = i[j - 1];
            } else if (beats(l, j)) {  // l lands here (slot j's old value moved down)
                v[j] = l;
                i[j] = e;
            }
        }
        if (beats(l, 0)) {
            v[0] = l;
            i[0] = e;
        }
    }
    // Slot j of the list (j compile-time after unrolling by the caller).
    __device__ __forceinline__ float value(int j) const {
        float r = v[0];
#pragma unroll
        for (int q = 1; q <= kMaxTopK; ++q)
            if (q == j) r = v[q];
        return r;
    }
    __device__ __forceinline__ int index(int j) const {
        int r = i[0];
#pragma unroll
        for (int q = 1; q <= kMaxTopK; ++q)
            if (q == j) r = i[q];
        return r;
    }
    // Slots left empty (only NaN logits were left) take the lowest indices
    // not selected yet, as a sequential scan would.
    __device__ __forceinline__ void fill_empty(int k) {
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k && i[j] < 0) {
                int e = 0;
                bool clash = true;
                while (clash) {
                    clash = false;
#pragma unroll
                    for (int q = 0; q < kMaxTopK; ++q)
                        if (q < j && i[q] == e) clash = true;
                    if (clash) ++e;
                }
                i[j] = e;
            }
        }
    }
};

// "a before b" in the selection order: non-empty before empty, larger value,
// then lower index.
__device__ __forceinline__ bool topk_before(float av, int ai, float bv, int bi) {
    if (ai < 0) return false;
    if (bi < 0) return true;
    return av > bv || (av == bv && ai < bi);
}

}  // namespace l4moe
