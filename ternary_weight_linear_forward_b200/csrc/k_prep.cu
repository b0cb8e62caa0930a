// k_prep.cu -- offline weight preparation: absmean scale, ternarisation and
// 2-bit packing; for the 1-bit variant, the mean, binarisation and 1-bit
// packing.
//
// absmean (DataCamp blog "MatMul-free language models", section "MatMul
// vervangen door ternaire bewerkingen"): divide the weight matrix by its mean
// absolute value and round each element to the nearest of -1, 0, +1.
//
// The mean is formed without any order dependence: pass 1 finds the largest
// |w| (an integer max over bit patterns), pass 2 turns every |w| into a 64-bit
// fixed-point integer on the grid set by that maximum and adds the integers
// exactly in 128 bits; the last CTA converts the exact integer sum to beta.
// Pass 3 divides and rounds.  All three passes stream W with 16-byte loads
// from a grid of a few CTAs per SM; they are HBM-bound and run once per matrix.
#include "common.cuh"
#include "kernels.cuh"

namespace bl {

namespace {

constexpr int PREP_THREADS = 256;

struct u128 {
    unsigned long long lo, hi;
};

__device__ __forceinline__ void add128(u128& a, unsigned long long lo, unsigned long long hi) {
    unsigned long long s = a.lo + lo;
    a.hi += hi + (s < lo ? 1ull : 0ull);
    a.lo = s;
}

__device__ __forceinline__ u128 shfl_xor128(u128 v, int off) {
    u128 r;
    r.lo = __shfl_xor_sync(0xffffffffu, v.lo, off);
    r.hi = __shfl_xor_sync(0xffffffffu, v.hi, off);
    return r;
}

// Fixed-point value of |w| on the grid 2^(E - 188), E = max(biased exponent
// of max|W|, 1): exact for exponents >= E - 38, truncated below, < 2^62.
__device__ __forceinline__ unsigned long long fixed_abs(uint32_t bits, int E) {
    uint32_t u = bits & 0x7FFFFFFFu;
    int e = (int)(u >> 23);
    unsigned long long m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    int ee = e ? e : 1;
    int sh = ee - E + 38;
    if (sh >= 0) return m << sh;
    if (sh <= -24) return 0ull;
    return m >> (-sh);
}

__global__ void __launch_bounds__(PREP_THREADS) absmax_bits_kernel(const float4* __restrict__ W, long long n4,
                                                                   unsigned* __restrict__ ws_max) {
    unsigned mx = 0;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float4 v = __ldg(&W[i]);
        mx = max(mx, __float_as_uint(v.x) & 0x7FFFFFFFu);
        mx = max(mx, __float_as_uint(v.y) & 0x7FFFFFFFu);
        mx = max(mx, __float_as_uint(v.z) & 0x7FFFFFFFu);
        mx = max(mx, __float_as_uint(v.w) & 0x7FFFFFFFu);
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    __shared__ unsigned sm[PREP_THREADS / 32];
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned v = threadIdx.x < PREP_THREADS / 32 ? sm[threadIdx.x] : 0u;
        v = __reduce_max_sync(0xffffffffu, v);
        if (threadIdx.x == 0) atomicMax(ws_max, v);
    }
}

// Correctly rounded conversion of a 128-bit unsigned integer to binary64.
__device__ double u128_to_double_rn(u128 s) {
    if (s.hi == 0) return __ull2double_rn(s.lo);
    int msb = 127 - __clzll((long long)s.hi);  // >= 64
    int sh = msb - 63;                         // 1 .. 64
    unsigned long long t, sticky;
    if (sh == 64) {
        t = s.hi;
        sticky = s.lo != 0;
    } else {
        t = (s.hi << (64 - sh)) | (s.lo >> sh);
        sticky = (s.lo << (64 - sh)) != 0;
    }
    // bit 0 of t lies 11 places below t's binary64 rounding position, so
    // OR-ing the sticky bit into it decides ties correctly.
    return scalbn(__ull2double_rn(t | sticky), sh);
}

__global__ void __launch_bounds__(PREP_THREADS) abssum_kernel(const float4* __restrict__ W, long long n4,
                                                              const unsigned* __restrict__ ws_max,
                                                              unsigned* __restrict__ ws_counter,
                                                              u128* __restrict__ partials, float* __restrict__ beta,
                                                              long long count) {
    const unsigned maxbits = *ws_max;
    const int E = max((int)(maxbits >> 23), 1);
    u128 acc = {0ull, 0ull};
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float4 v = __ldg(&W[i]);
        add128(acc, fixed_abs(__float_as_uint(v.x), E), 0);
        add128(acc, fixed_abs(__float_as_uint(v.y), E), 0);
        add128(acc, fixed_abs(__float_as_uint(v.z), E), 0);
        add128(acc, fixed_abs(__float_as_uint(v.w), E), 0);
    }
    for (int off = 16; off; off >>= 1) {
        u128 o = shfl_xor128(acc, off);
        add128(acc, o.lo, o.hi);
    }
    __shared__ u128 sm[PREP_THREADS / 32];
    __shared__ bool is_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sm[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        u128 t = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) add128(t, sm[w].lo, sm[w].hi);
        partials[blockIdx.x] = t;
        __threadfence();
        unsigned done = atomicAdd(ws_counter, 1u);
        is_last = (done == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // Last CTA: exact integer sum of all partials, then beta.
    u128 t = {0ull, 0ull};
    for (int b = threadIdx.x; b < (int)gridDim.x; b += blockDim.x) {
        u128 p;
        p.lo = __ldcg(&partials[b].lo);
        p.hi = __ldcg(&partials[b].hi);
        add128(t, p.lo, p.hi);
    }
    for (int off = 16; off; off >>= 1) {
        u128 o = shfl_xor128(t, off);
        add128(t, o.lo, o.hi);
    }
    __syncthreads();
    if (lane == 0) sm[warp] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
        u128 s = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) add128(s, sm[w].lo, sm[w].hi);
        double sum = scalbn(u128_to_double_rn(s), E - 188);
        *beta = __double2float_rn(__ddiv_rn(sum, (double)count));
        *ws_counter = 0u;
    }
}

__device__ __forceinline__ int8_t ternary_code(float w, float den) {
    float r = rintf(__fdiv_rn(w, den));
    r = fminf(fmaxf(r, -1.0f), 1.0f);
    return (int8_t)(int)r;
}

__global__ void __launch_bounds__(PREP_THREADS) ternarize_kernel(const float4* __restrict__ W, long long n4,
                                                                 const float* __restrict__ beta, float eps,
                                                                 char4* __restrict__ W_t) {
    const float den = __fadd_rn(*beta, eps);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float4 v = __ldg(&W[i]);
        char4 o;
        o.x = ternary_code(v.x, den);
        o.y = ternary_code(v.y, den);
        o.z = ternary_code(v.z, den);
        o.w = ternary_code(v.w, den);
        W_t[i] = o;
    }
}

// One thread per packed word: the 16 int8 trits of k = 16j .. 16j+15 are the
// 16 bytes at offset 16 * (flat word index) of W_t.
__global__ void __launch_bounds__(PREP_THREADS) pack_kernel(const int4* __restrict__ W_t, long long nwords,
                                                            uint32_t* __restrict__ W_p) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nwords;
         i += (long long)gridDim.x * blockDim.x) {
        int4 q = __ldg(&W_t[i]);
        // per byte: code = (w + 1) & 3 maps 0xFF/0/1 to 0/1/2 with no carry out
        uint32_t c0 = (((uint32_t)q.x & 0x03030303u) + 0x01010101u) & 0x03030303u;  // k = 16j + 0..3
        uint32_t c1 = (((uint32_t)q.y & 0x03030303u) + 0x01010101u) & 0x03030303u;  // k = 16j + 4..7
        uint32_t c2 = (((uint32_t)q.z & 0x03030303u) + 0x01010101u) & 0x03030303u;
        uint32_t c3 = (((uint32_t)q.w & 0x03030303u) + 0x01010101u) & 0x03030303u;
        W_p[i] = c0 | (c1 << 2) | (c2 << 4) | (c3 << 6);
    }
}

// ----------------------------------------------------------- 1-bit variant
//
// unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle
// auf lokale Geraete", "Mathematische Grundlagen", item 1
// "Gewichtsbinarisierung", eq. 1: W_b = Sign(W - alpha), alpha = mean(W),
// Sign(d) = +1 for d > 0, -1 otherwise.  beta stays the absmean scale.
//
// The sums pass keeps two exact fixed-point integers per thread, one for the
// positive and one for the negative elements (same grid as above): their sum
// gives sum |W| (beta) and their difference the signed sum (alpha), each
// rounded once to binary64 by the last CTA.

__global__ void __launch_bounds__(PREP_THREADS) signed_sums_kernel(const float4* __restrict__ W, long long n4,
                                                                   const unsigned* __restrict__ ws_max,
                                                                   unsigned* __restrict__ ws_counter,
                                                                   u128* __restrict__ partials,
                                                                   float* __restrict__ alpha,
                                                                   float* __restrict__ beta, long long count) {
    const unsigned maxbits = *ws_max;
    const int E = max((int)(maxbits >> 23), 1);
    u128 pos = {0ull, 0ull}, neg = {0ull, 0ull};
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        const float4 v = __ldg(&W[i]);
        const uint32_t b[4] = {__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                               __float_as_uint(v.w)};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const unsigned long long f = fixed_abs(b[j], E);
            if (b[j] >> 31)
                add128(neg, f, 0);
            else
                add128(pos, f, 0);
        }
    }
    for (int off = 16; off; off >>= 1) {
        u128 o = shfl_xor128(pos, off);
        add128(pos, o.lo, o.hi);
        o = shfl_xor128(neg, off);
        add128(neg, o.lo, o.hi);
    }
    __shared__ u128 sp[PREP_THREADS / 32], sn[PREP_THREADS / 32];
    __shared__ bool is_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sp[warp] = pos;
        sn[warp] = neg;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        u128 tp = {0ull, 0ull}, tn = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) {
            add128(tp, sp[w].lo, sp[w].hi);
            add128(tn, sn[w].lo, sn[w].hi);
        }
        partials[2 * blockIdx.x] = tp;
        partials[2 * blockIdx.x + 1] = tn;
        __threadfence();
        unsigned done = atomicAdd(ws_counter, 1u);
        is_last = (done == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // Last CTA: exact totals of both integers, then alpha and beta.
    u128 tp = {0ull, 0ull}, tn = {0ull, 0ull};
    for (int b = threadIdx.x; b < (int)gridDim.x; b += blockDim.x) {
        add128(tp, __ldcg(&partials[2 * b].lo), __ldcg(&partials[2 * b].hi));
        add128(tn, __ldcg(&partials[2 * b + 1].lo), __ldcg(&partials[2 * b + 1].hi));
    }
    for (int off = 16; off; off >>= 1) {
        u128 o = shfl_xor128(tp, off);
        add128(tp, o.lo, o.hi);
        o = shfl_xor128(tn, off);
        add128(tn, o.lo, o.hi);
    }
    __syncthreads();
    if (lane == 0) {
        sp[warp] = tp;
        sn[warp] = tn;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        u128 P = {0ull, 0ull}, Q = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) {
            add128(P, sp[w].lo, sp[w].hi);
            add128(Q, sn[w].lo, sn[w].hi);
        }
        u128 A = P;  // P + Q < 2^127: no carry out
        add128(A, Q.lo, Q.hi);
        const bool neg_sum = Q.hi > P.hi || (Q.hi == P.hi && Q.lo > P.lo);
        const u128& big = neg_sum ? Q : P;
        const u128& small = neg_sum ? P : Q;
        u128 D;  // |P - Q|
        D.lo = big.lo - small.lo;
        D.hi = big.hi - small.hi - (big.lo < small.lo ? 1ull : 0ull);
        const double abs_sum = scalbn(u128_to_double_rn(A), E - 188);
        double sum = scalbn(u128_to_double_rn(D), E - 188);
        if (neg_sum) sum = -sum;
        *beta = __double2float_rn(__ddiv_rn(abs_sum, (double)count));
        *alpha = __double2float_rn(__ddiv_rn(sum, (double)count));
        *ws_counter = 0u;
    }
}

__global__ void __launch_bounds__(PREP_THREADS) binarize_kernel(const float4* __restrict__ W, long long n4,
                                                                const float* __restrict__ alpha,
                                                                char4* __restrict__ W_b) {
    const float a = *alpha;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        const float4 v = __ldg(&W[i]);
        char4 o;  // Sign(w - alpha), Sign(0) = -1
        o.x = __fsub_rn(v.x, a) > 0.0f ? 1 : -1;
        o.y = __fsub_rn(v.y, a) > 0.0f ? 1 : -1;
        o.z = __fsub_rn(v.z, a) > 0.0f ? 1 : -1;
        o.w = __fsub_rn(v.w, a) > 0.0f ? 1 : -1;
        W_b[i] = o;
    }
}

// One thread per packed word: the 32 int8 weights of k = 32j .. 32j+31 are
// the 32 bytes at offset 32 * (flat word index) of W_b.  Byte b of int s
// (k = 32j + 4s + b) becomes bit 8b + s, set when the weight is > 0.
__global__ void __launch_bounds__(PREP_THREADS) pack_bits_kernel(const int4* __restrict__ W_b, long long nwords,
                                                                 uint32_t* __restrict__ W_p) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nwords;
         i += (long long)gridDim.x * blockDim.x) {
        const int4 lo = __ldg(&W_b[2 * i]), hi = __ldg(&W_b[2 * i + 1]);
        const uint32_t v[8] = {(uint32_t)lo.x, (uint32_t)lo.y, (uint32_t)lo.z, (uint32_t)lo.w,
                               (uint32_t)hi.x, (uint32_t)hi.y, (uint32_t)hi.z, (uint32_t)hi.w};
        uint32_t word = 0;
#pragma unroll
        for (int s = 0; s < 8; ++s) word |= (__vcmpgts4(v[s], 0u) & 0x01010101u) << s;
        W_p[i] = word;
    }
}

}  // namespace

size_t binarize_weights_ws_bytes() { return 256 + 2 * sizeof(u128) * (size_t)PREP_MAX_GRID; }

cudaError_t launch_binarize_weights(const float* W, long long n, int8_t* W_b, float* alpha, float* beta, void* ws,
                                    int num_sms, cudaStream_t st) {
    unsigned* ws_max = reinterpret_cast<unsigned*>(ws);
    unsigned* ws_counter = ws_max + 1;
    u128* partials = reinterpret_cast<u128*>(reinterpret_cast<char*>(ws) + 256);
    const long long n4 = n / 4;
    const long long want = (n4 + PREP_THREADS - 1) / PREP_THREADS;
    int grid = (int)std::min<long long>(std::min<long long>(want, (long long)num_sms * 4), PREP_MAX_GRID);
    grid = std::max(grid, 1);
    cudaError_t e = cudaMemsetAsync(ws, 0, 16, st);
    if (e != cudaSuccess) return e;
    const float4* W4 = reinterpret_cast<const float4*>(W);
    absmax_bits_kernel<<<grid, PREP_THREADS, 0, st>>>(W4, n4, ws_max);
    signed_sums_kernel<<<grid, PREP_THREADS, 0, st>>>(W4, n4, ws_max, ws_counter, partials, alpha, beta, n);
    binarize_kernel<<<grid, PREP_THREADS, 0, st>>>(W4, n4, alpha, reinterpret_cast<char4*>(W_b));
    return cudaGetLastError();
}

cudaError_t launch_pack_bits(const int8_t* W_b, long long nwords, uint32_t* W_p, int num_sms, cudaStream_t st) {
    const long long want = (nwords + PREP_THREADS - 1) / PREP_THREADS;
    const int grid = (int)std::max<long long>(1, std::min<long long>(want, (long long)num_sms * 8));
    pack_bits_kernel<<<grid, PREP_THREADS, 0, st>>>(reinterpret_cast<const int4*>(W_b), nwords, W_p);
    return cudaGetLastError();
}

size_t quantize_weights_ws_bytes() { return 256 + sizeof(u128) * (size_t)PREP_MAX_GRID; }

cudaError_t launch_quantize_weights(const float* W, long long n, float eps, int8_t* W_t, float* beta, void* ws,
                                    int num_sms, cudaStream_t st) {
    unsigned* ws_max = reinterpret_cast<unsigned*>(ws);
    unsigned* ws_counter = ws_max + 1;
    u128* partials = reinterpret_cast<u128*>(reinterpret_cast<char*>(ws) + 256);
    long long n4 = n / 4;
    long long want = (n4 + PREP_THREADS - 1) / PREP_THREADS;
    int grid = (int)std::min<long long>(std::min<long long>(want, (long long)num_sms * 4), PREP_MAX_GRID);
    grid = std::max(grid, 1);
    cudaError_t e = cudaMemsetAsync(ws, 0, 16, st);
    if (e != cudaSuccess) return e;
    absmax_bits_kernel<<<grid, PREP_THREADS, 0, st>>>(reinterpret_cast<const float4*>(W), n4, ws_max);
    abssum_kernel<<<grid, PREP_THREADS, 0, st>>>(reinterpret_cast<const float4*>(W), n4, ws_max, ws_counter, partials,
                                                 beta, n);
    ternarize_kernel<<<grid, PREP_THREADS, 0, st>>>(reinterpret_cast<const float4*>(W), n4, beta, eps,
                                                    reinterpret_cast<char4*>(W_t));
    return cudaGetLastError();
}

cudaError_t launch_pack(const int8_t* W_t, long long nwords, uint32_t* W_p, int num_sms, cudaStream_t st) {
    long long want = (nwords + PREP_THREADS - 1) / PREP_THREADS;
    int grid = (int)std::max<long long>(1, std::min<long long>(want, (long long)num_sms * 8));
    pack_kernel<<<grid, PREP_THREADS, 0, st>>>(reinterpret_cast<const int4*>(W_t), nwords, W_p);
    return cudaGetLastError();
}

}  // namespace bl
