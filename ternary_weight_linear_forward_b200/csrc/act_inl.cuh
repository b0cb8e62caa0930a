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

// rint(x * s) clamped to [-127, 127], as the standalone quantiser.  Adding
// 1.5 * 2^23 rounds the binary32 product to an integer, ties to even, exactly
// like rint, because |x * s| <= 127 (1 + 2^-22) is far below 2^22; the integer
// is then the low bits of the sum.  (An FADD on the FMA pipe instead of a
// conversion on the quarter-rate XU pipe.)
__device__ __forceinline__ int q8(float v, float s) {
    const float t = __fadd_rn(__fmul_rn(v, s), 12582912.0f);
    const int r = __float_as_int(t) - 0x4B400000;
    return min(max(r, -127), 127);
}

// One 16-element chunk of an activation row in its storage format:
// 4 x 16 bytes of fp32, 2 x 16 bytes of bf16 or 16 int8 codes.
template <int XM>
struct XChunk {
    uint4 u[XM == X_F32 ? 4 : (XM == X_BF16 ? 2 : 1)];
};

// chunk g of `row` (read-only path)
template <int XM>
__device__ __forceinline__ void ld_chunk(const void* row, int g, XChunk<XM>& c) {
    constexpr int n = XM == X_F32 ? 4 : (XM == X_BF16 ? 2 : 1);
    const uint4* pp = reinterpret_cast<const uint4*>(row) + n * g;
#pragma unroll
    for (int i = 0; i < n; ++i) c.u[i] = __ldg(pp + i);
}

// the chunk's 16 values as binary32 (X_F32 or X_BF16)
template <int XM>
__device__ __forceinline__ void cvt_chunk(const XChunk<XM>& c, float (&v)[16]) {
    if constexpr (XM == X_BF16) {
        const uint32_t w[8] = {c.u[0].x, c.u[0].y, c.u[0].z, c.u[0].w, c.u[1].x, c.u[1].y, c.u[1].z, c.u[1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[4 * i] = __uint_as_float(c.u[i].x);
            v[4 * i + 1] = __uint_as_float(c.u[i].y);
            v[4 * i + 2] = __uint_as_float(c.u[i].z);
            v[4 * i + 3] = __uint_as_float(c.u[i].w);
        }
    }
}

template <int MODE>  // X_F32 or X_BF16
__device__ __forceinline__ void load16(const void* row, int g, float (&v)[16]) {
    XChunk<MODE> c;
    ld_chunk<MODE>(row, g, c);
    cvt_chunk<MODE>(c, v);
}

// max |v| over the chunk, as the bit pattern of a non-negative float
template <int XM>
__device__ __forceinline__ unsigned chunk_absmax(const XChunk<XM>& c, unsigned a) {
    float v[16];
    cvt_chunk<XM>(c, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) a = max(a, __float_as_uint(fabsf(v[i])));
    return a;
}

// the chunk's 16 int8 codes (quantised with scale s unless already int8)
template <int XM>
__device__ __forceinline__ int4 chunk_codes(const XChunk<XM>& c, float s) {
    if constexpr (XM == X_QUANTISED) {
        return make_int4((int)c.u[0].x, (int)c.u[0].y, (int)c.u[0].z, (int)c.u[0].w);
    } else {
        float v[16];
        cvt_chunk<XM>(c, v);
        int4 q;
        q.x = (int)pack4(q8(v[0], s), q8(v[1], s), q8(v[2], s), q8(v[3], s));
        q.y = (int)pack4(q8(v[4], s), q8(v[5], s), q8(v[6], s), q8(v[7], s));
        q.z = (int)pack4(q8(v[8], s), q8(v[9], s), q8(v[10], s), q8(v[11], s));
        q.w = (int)pack4(q8(v[12], s), q8(v[13], s), q8(v[14], s), q8(v[15], s));
        return q;
    }
}

}  // namespace bl
