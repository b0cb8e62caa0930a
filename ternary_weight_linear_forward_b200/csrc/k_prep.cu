// k_prep.cu -- offline weight preparation: absmean scale, ternarisation and
// 2-bit packing; for the 1-bit variant, the mean, binarisation and 1-bit
// packing.
//
// absmean (DataCamp blog "MatMul-free language models", section "MatMul
// vervangen door ternaire bewerkingen"): divide the weight matrix by its mean
// absolute value and round each element to the nearest of -1, 0, +1.
//
// The mean is formed exactly, without any order dependence, over the whole
// binary32 range: pass 1 finds the largest |w| (an integer max over bit
// patterns), pass 2 adds every |w| exactly.  An element within 2^38 of the
// maximum is a 64-bit fixed-point integer on the grid 2^(E - 188) set by that
// maximum and goes into a per-thread 128-bit sum; a smaller one (rare) is an
// integer on the grid 2^-149 of the smallest subnormal and goes, by its
// exponent block of 16, into one of sixteen 128-bit sums of the CTA in
// shared memory.  The last CTA adds all partial sums exactly, assembles them
// into one multi-word integer and rounds it once to binary64 (then beta =
// that / count, rounded to binary64, then to binary32).  Pass 3 divides and
// rounds.  All three passes stream W with 16-byte loads from a grid of a few
// CTAs per SM; they are HBM-bound and run once per matrix.
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

// Exponent blocks of the small-element sums: |w| = m 2^(ee - 150) with
// ee - 1 in [0, 253] is the integer m 2^(ee - 1) on the grid 2^-149; block
// b = (ee - 1) / 16 holds m 2^((ee - 1) % 16) < 2^40 per element.
constexpr int SMALL_BLOCKS = 16;
constexpr int SMALL_BITS = 16;

// The CTA's small-element sums (shared memory), 128 bits each, kept by
// 64-bit atomics: a carry out of the low word adds one to the high word.
struct SmallSums {
    unsigned long long lo[SMALL_BLOCKS], hi[SMALL_BLOCKS];
};

__device__ __forceinline__ void small_sums_clear(SmallSums& s) {
    if (threadIdx.x < SMALL_BLOCKS) s.lo[threadIdx.x] = s.hi[threadIdx.x] = 0ull;
}

// Add |w| (bit pattern `bits`) exactly: to the thread's 128-bit sum on the
// grid 2^(E - 188) when its exponent is at least E - 38 (E = max(biased
// exponent of max|W|, 1); the value is then < 2^62 there), else to the CTA's
// small-element sum of its exponent block.
__device__ __forceinline__ void exact_abs_add(uint32_t bits, int E, u128& fast, SmallSums& small) {
    const uint32_t u = bits & 0x7FFFFFFFu;
    const int e = (int)(u >> 23);
    const unsigned long long m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    if (m == 0ull) return;
    const int ee = e ? e : 1;
    const int sh = ee - E + 38;
    if (sh >= 0) {
        add128(fast, m << sh, 0ull);
        return;
    }
    const int t = ee - 1;
    const unsigned long long v = m << (t % SMALL_BITS);
    const unsigned long long old = atomicAdd(&small.lo[t / SMALL_BITS], v);
    if (old + v < old) atomicAdd(&small.hi[t / SMALL_BITS], 1ull);
}

// A nonnegative integer of up to 24 * 32 bits: word i holds bits [32i, 32i + 32)
// once normalised; before that each word is a 64-bit sum of 32-bit pieces.
struct Big {
    unsigned long long w[24];
};

__device__ void big_clear(Big& a) {
    for (int i = 0; i < 24; ++i) a.w[i] = 0ull;
}

// a += v * 2^shift (0 <= shift <= 600)
__device__ void big_add(Big& a, u128 v, int shift) {
    const unsigned long long piece[4] = {v.lo & 0xFFFFFFFFull, v.lo >> 32, v.hi & 0xFFFFFFFFull, v.hi >> 32};
    for (int k = 0; k < 4; ++k) {
        const int pos = shift + 32 * k;
        const unsigned long long x = piece[k] << (pos & 31);  // < 2^63
        a.w[pos >> 5] += x & 0xFFFFFFFFull;
        a.w[(pos >> 5) + 1] += x >> 32;
    }
}

__device__ void big_normalise(Big& a) {
    for (int i = 0; i < 23; ++i) {
        a.w[i + 1] += a.w[i] >> 32;
        a.w[i] &= 0xFFFFFFFFull;
    }
}

// bits [lo, lo + 64) of a normalised Big (lo >= 0)
__device__ unsigned long long big_bits64(const Big& a, int lo) {
    const int L = lo >> 5, o = lo & 31;
    unsigned long long t = a.w[L] >> o;
    if (L + 1 < 24) t |= a.w[L + 1] << (32 - o);
    if (L + 2 < 24 && o) t |= a.w[L + 2] << (64 - o);
    return t;
}

// Correctly rounded binary64 value of a normalised Big times 2^unit_exp.
__device__ double big_to_double_rn(const Big& a, int unit_exp) {
    int top = 23;
    while (top >= 0 && a.w[top] == 0ull) --top;
    if (top < 0) return 0.0;
    const int msb = 32 * top + 31 - __clzll((long long)a.w[top]) + 32;  // bit index of the leading one
    const int lsb = msb - 63;
    if (lsb <= 0) return scalbn(__ull2double_rn(big_bits64(a, 0)), unit_exp);
    unsigned long long t = big_bits64(a, lsb);
    // bit 0 of t lies 11 places below t's binary64 rounding position, so
    // OR-ing the sticky bit into it decides ties correctly
    bool sticky = (a.w[lsb >> 5] & ((1ull << (lsb & 31)) - 1ull)) != 0ull;
    for (int i = 0; i < (lsb >> 5); ++i) sticky = sticky || a.w[i] != 0ull;
    return scalbn(__ull2double_rn(t | (sticky ? 1ull : 0ull)), lsb + unit_exp);
}

// The exact sum as a Big and the exponent of its unit: the fast sum F on the
// grid 2^(E - 188) and the small-element block sums S_b (grid 2^-149, block
// b shifted by 16 b).  When E < 39 every element is on the fast grid, which
// is then the finer one.
__device__ void exact_total(u128 F, const u128* S, int E, Big& out, int& unit_exp) {
    big_clear(out);
    if (E < 39) {
        big_add(out, F, 0);
        unit_exp = E - 188;
    } else {
        big_add(out, F, E - 39);
        for (int b = 0; b < SMALL_BLOCKS; ++b) big_add(out, S[b], SMALL_BITS * b);
        unit_exp = -149;
    }
    big_normalise(out);
}

// Sum over the grid's CTAs of the small-element partials (SMALL_BLOCKS u128
// per CTA at `part`, CTA stride `stride` u128): thread t < SMALL_BLOCKS ends
// with block t's total in tot.  Called by every thread of the last CTA.
__device__ void small_partials_total(const u128* part, int stride, int nblocks, u128 (&red)[SMALL_BLOCKS][16],
                                     u128& tot) {
    const int b = threadIdx.x % SMALL_BLOCKS, slot = threadIdx.x / SMALL_BLOCKS;  // 256 threads: 16 slots
    u128 t = {0ull, 0ull};
    for (int g = slot; g < nblocks; g += 16)
        add128(t, __ldcg(&part[(size_t)g * stride + b].lo), __ldcg(&part[(size_t)g * stride + b].hi));
    red[b][slot] = t;
    __syncthreads();
    tot = {0ull, 0ull};
    if (threadIdx.x < SMALL_BLOCKS)
        for (int s = 0; s < 16; ++s) add128(tot, red[threadIdx.x][s].lo, red[threadIdx.x][s].hi);
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

// partials: per CTA one u128 fast sum followed by SMALL_BLOCKS u128 small sums
__global__ void __launch_bounds__(PREP_THREADS) abssum_kernel(const float4* __restrict__ W, long long n4,
                                                              const unsigned* __restrict__ ws_max,
                                                              unsigned* __restrict__ ws_counter,
                                                              u128* __restrict__ partials, float* __restrict__ beta,
                                                              long long count) {
    constexpr int STRIDE = 1 + SMALL_BLOCKS;
    __shared__ SmallSums small;
    small_sums_clear(small);
    __syncthreads();
    const unsigned maxbits = *ws_max;
    const int E = max((int)(maxbits >> 23), 1);
    u128 acc = {0ull, 0ull};
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4;
         i += (long long)gridDim.x * blockDim.x) {
        float4 v = __ldg(&W[i]);
        exact_abs_add(__float_as_uint(v.x), E, acc, small);
        exact_abs_add(__float_as_uint(v.y), E, acc, small);
        exact_abs_add(__float_as_uint(v.z), E, acc, small);
        exact_abs_add(__float_as_uint(v.w), E, acc, small);
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
    if (threadIdx.x < SMALL_BLOCKS)
        partials[(size_t)blockIdx.x * STRIDE + 1 + threadIdx.x] = {small.lo[threadIdx.x], small.hi[threadIdx.x]};
    if (threadIdx.x == 0) {
        u128 t = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) add128(t, sm[w].lo, sm[w].hi);
        partials[(size_t)blockIdx.x * STRIDE] = t;
    }
    __threadfence();  // every writer's partials are visible before the CTA is counted
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned done = atomicAdd(ws_counter, 1u);
        is_last = (done == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // Last CTA: exact integer sums of all partials, then beta.
    __shared__ u128 red[SMALL_BLOCKS][16];
    __shared__ u128 small_tot[SMALL_BLOCKS];
    u128 st;
    small_partials_total(partials + 1, STRIDE, (int)gridDim.x, red, st);
    if (threadIdx.x < SMALL_BLOCKS) small_tot[threadIdx.x] = st;
    u128 t = {0ull, 0ull};
    for (int b = threadIdx.x; b < (int)gridDim.x; b += blockDim.x) {
        u128 p;
        p.lo = __ldcg(&partials[(size_t)b * STRIDE].lo);
        p.hi = __ldcg(&partials[(size_t)b * STRIDE].hi);
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
        Big total;
        int unit_exp;
        exact_total(s, small_tot, E, total, unit_exp);
        const double sum = big_to_double_rn(total, unit_exp);
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
    // partials: per CTA the positive then the negative sums, each one u128
    // fast sum followed by SMALL_BLOCKS u128 small sums
    constexpr int STRIDE = 1 + SMALL_BLOCKS;
    __shared__ SmallSums small_p, small_n;
    small_sums_clear(small_p);
    small_sums_clear(small_n);
    __syncthreads();
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
            if (b[j] >> 31)
                exact_abs_add(b[j], E, neg, small_n);
            else
                exact_abs_add(b[j], E, pos, small_p);
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
    u128* const mine = partials + (size_t)blockIdx.x * 2 * STRIDE;
    if (threadIdx.x < SMALL_BLOCKS) {
        mine[1 + threadIdx.x] = {small_p.lo[threadIdx.x], small_p.hi[threadIdx.x]};
        mine[STRIDE + 1 + threadIdx.x] = {small_n.lo[threadIdx.x], small_n.hi[threadIdx.x]};
    }
    if (threadIdx.x == 0) {
        u128 tp = {0ull, 0ull}, tn = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) {
            add128(tp, sp[w].lo, sp[w].hi);
            add128(tn, sn[w].lo, sn[w].hi);
        }
        mine[0] = tp;
        mine[STRIDE] = tn;
    }
    __threadfence();  // every writer's partials are visible before the CTA is counted
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned done = atomicAdd(ws_counter, 1u);
        is_last = (done == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // Last CTA: exact totals of both integers, then alpha and beta.
    __shared__ u128 red[SMALL_BLOCKS][16];
    __shared__ u128 small_tp[SMALL_BLOCKS], small_tn[SMALL_BLOCKS];
    u128 st;
    small_partials_total(partials + 1, 2 * STRIDE, (int)gridDim.x, red, st);
    if (threadIdx.x < SMALL_BLOCKS) small_tp[threadIdx.x] = st;
    __syncthreads();
    small_partials_total(partials + STRIDE + 1, 2 * STRIDE, (int)gridDim.x, red, st);
    if (threadIdx.x < SMALL_BLOCKS) small_tn[threadIdx.x] = st;
    u128 tp = {0ull, 0ull}, tn = {0ull, 0ull};
    for (int b = threadIdx.x; b < (int)gridDim.x; b += blockDim.x) {
        const u128* p = partials + (size_t)b * 2 * STRIDE;
        add128(tp, __ldcg(&p[0].lo), __ldcg(&p[0].hi));
        add128(tn, __ldcg(&p[STRIDE].lo), __ldcg(&p[STRIDE].hi));
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
        u128 fp = {0ull, 0ull}, fn = {0ull, 0ull};
        for (int w = 0; w < PREP_THREADS / 32; ++w) {
            add128(fp, sp[w].lo, sp[w].hi);
            add128(fn, sn[w].lo, sn[w].hi);
        }
        Big P, Q, A, D;
        int unit_exp;
        exact_total(fp, small_tp, E, P, unit_exp);
        exact_total(fn, small_tn, E, Q, unit_exp);
        int top = 23;  // compare P and Q from the top word
        while (top > 0 && P.w[top] == Q.w[top]) --top;
        const bool neg_sum = Q.w[top] > P.w[top];
        const Big& hi = neg_sum ? Q : P;
        const Big& lo = neg_sum ? P : Q;
        unsigned long long borrow = 0ull;
        for (int i = 0; i < 24; ++i) {  // A = P + Q, D = |P - Q| (normalised words)
            A.w[i] = P.w[i] + Q.w[i];
            const unsigned long long d = hi.w[i] - lo.w[i] - borrow;
            borrow = hi.w[i] < lo.w[i] + borrow ? 1ull : 0ull;
            D.w[i] = d & 0xFFFFFFFFull;
        }
        big_normalise(A);
        const double abs_sum = big_to_double_rn(A, unit_exp);
        double sum = big_to_double_rn(D, unit_exp);
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

size_t binarize_weights_ws_bytes() { return 256 + 2 * (1 + SMALL_BLOCKS) * sizeof(u128) * (size_t)PREP_MAX_GRID; }

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

size_t quantize_weights_ws_bytes() { return 256 + (1 + SMALL_BLOCKS) * sizeof(u128) * (size_t)PREP_MAX_GRID; }

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
