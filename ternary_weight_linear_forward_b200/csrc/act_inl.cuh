// act_inl.cuh -- per-token absmax int8 quantisation helpers shared by the
// decode kernels that quantise their activations in the prologue.
//
// unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle
// auf lokale Geraete", "Mathematische Grundlagen", eq. 2
// "Aktivierungsquantisierung": gamma = ||x||_inf per token, Q_b = 127; the
// code is rint(x * (127 / gamma)) clamped to [-127, 127], the same rounding as
// the standalone quantiser kernel.
#pragma once

#include "common.cuh"

namespace bl {

// How a decode kernel receives its activations.
enum XMode : int { X_QUANTISED = 0, X_F32 = 1, X_BF16 = 2 };

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
           ((uint32_t)(d & 0xFF) << 24);
}

// same rounding as the standalone quantiser: rint(x * s), clamp to [-127, 127]
__device__ __forceinline__ int q8(float v, float s) {
    int r = __float2int_rn(__fmul_rn(v, s));
    return min(max(r, -127), 127);
}

template <int MODE>  // X_F32 or X_BF16
__device__ __forceinline__ void load16(const void* row, int g, float (&v)[16]) {
    if (MODE == X_BF16) {
        const uint4* pp = reinterpret_cast<const uint4*>(row) + 2 * g;
        uint4 a = __ldg(pp), b = __ldg(pp + 1);
        uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
        const float4* pp = reinterpret_cast<const float4*>(row) + 4 * g;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 f = __ldg(pp + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
    }
}

}  // namespace bl
