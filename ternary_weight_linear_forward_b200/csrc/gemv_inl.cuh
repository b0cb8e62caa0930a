// gemv_inl.cuh -- inner steps of the CUDA-core decode kernels: the masked
// dp4a contraction of packed trits and the batched warp reduction.
//
// DataCamp blog "MatMul-free language models", section "MatMul vervangen
// door ternaire bewerkingen": each weight is -1, 0 or +1, so the dot product
// is an integer accumulation.  The packed code of k = 16j + 4s + b is
// c = w + 1 at bits 8b + 2s of word j.
#pragma once

#include "common.cuh"

namespace bl {

// 4^s-weighted accumulation of the 16 trits of word w against 16 x bytes
// held as x0..x3 (k = 16j + 4s .. 16j + 4s + 3 in x_s).
__device__ __forceinline__ void word_dot(uint32_t w, int x0, int x1, int x2, int x3, int& a0, int& a1, int& a2,
                                         int& a3) {
    a0 = dp4a_us(w & 0x03030303u, x0, a0);
    a1 = dp4a_us(w & 0x0C0C0C0Cu, x1, a1);
    a2 = dp4a_us(w & 0x30303030u, x2, a2);
    a3 = dp4a_us(w & 0xC0C0C0C0u, x3, a3);
}

__device__ __forceinline__ int combine4(int a0, int a1, int a2, int a3) {
    return a0 + (a1 >> 2) + (a2 >> 4) + (a3 >> 6);  // each a_s is a multiple of 4^s
}

// Batched reduction of V = 1, 2 or 4 values over the LPR lanes of a team.
// Lane tl ends up with the full sum of value `which`.
template <int LPR, int V>
__device__ __forceinline__ int team_reduce(const int (&v)[V], int tl, int& which) {
    if constexpr (V == 1) {
        int k = v[0];
#pragma unroll
        for (int o = LPR / 2; o; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
        which = 0;
        return k;
    } else if constexpr (V == 2) {
        constexpr int h1 = LPR / 2;
        const bool hi = (tl & h1) != 0;
        int k = hi ? v[1] : v[0];
        k += __shfl_xor_sync(0xffffffffu, hi ? v[0] : v[1], h1);
#pragma unroll
        for (int o = LPR / 4; o; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
        which = hi ? 1 : 0;
        return k;
    } else {
        constexpr int h1 = LPR / 2, h2 = LPR / 4;
        const bool hi = (tl & h1) != 0;
        int k0 = hi ? v[2] : v[0];
        int k1 = hi ? v[3] : v[1];
        k0 += __shfl_xor_sync(0xffffffffu, hi ? v[0] : v[2], h1);
        k1 += __shfl_xor_sync(0xffffffffu, hi ? v[1] : v[3], h1);
        const bool hi2 = (tl & h2) != 0;
        int k = hi2 ? k1 : k0;
        k += __shfl_xor_sync(0xffffffffu, hi2 ? k0 : k1, h2);
#pragma unroll
        for (int o = LPR / 8; o; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
        which = (hi ? 2 : 0) + (hi2 ? 1 : 0);
        return k;
    }
}

}  // namespace bl
