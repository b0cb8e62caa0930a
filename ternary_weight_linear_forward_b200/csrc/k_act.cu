// k_act.cu -- per-token absmax int8 activation quantisers.
//
// unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle
// auf lokale Geraete", "Mathematische Grundlagen", eq. 2
// "Aktivierungsquantisierung": x_hat = Clip(x * Q_b / gamma, ...), gamma =
// ||x||_inf.  Here Q_b = 127, gamma is per token and floored at 1e-5, the
// scale s = 127 / gamma is formed first (IEEE divide) and x * s is rounded to
// nearest-even and clamped to [-127, 127].
//
// One CTA per token row: pass 1 reduces max |x| (and, for the RMSNorm form,
// sum x^2 in binary64), pass 2 re-reads the row from L1/L2 and writes 16
// codes per thread per step with one 16-byte store.
#include "common.cuh"
#include "kernels.cuh"

namespace bl {

namespace {

constexpr int ACT_THREADS = 256;

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
           ((uint32_t)(d & 0xFF) << 24);
}

__device__ __forceinline__ int q8(float v, float s) {
    int r = __float2int_rn(__fmul_rn(v, s));
    return min(max(r, -127), 127);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16 consecutive activations of group g (k = 16g .. 16g+15) as fp32.
template <bool BF16>
__device__ __forceinline__ void load16(const void* row, int g, float (&v)[16]) {
    if (BF16) {
        const uint4* p = reinterpret_cast<const uint4*>(row) + 2 * g;
        uint4 a = __ldg(p), b = __ldg(p + 1);
        uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = bf16lo(w[i]);
            v[2 * i + 1] = bf16hi(w[i]);
        }
    } else {
        const float4* p = reinterpret_cast<const float4*>(row) + 4 * g;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 f = __ldg(p + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
    }
}

// Returns the sum of the 16 codes.
__device__ __forceinline__ int store16(int8_t* row_q, int g, const float (&v)[16], float s) {
    uint4 o;
    o.x = pack4(q8(v[0], s), q8(v[1], s), q8(v[2], s), q8(v[3], s));
    o.y = pack4(q8(v[4], s), q8(v[5], s), q8(v[6], s), q8(v[7], s));
    o.z = pack4(q8(v[8], s), q8(v[9], s), q8(v[10], s), q8(v[11], s));
    o.w = pack4(q8(v[12], s), q8(v[13], s), q8(v[14], s), q8(v[15], s));
    reinterpret_cast<uint4*>(row_q)[g] = o;
    return __dp4a((int)o.x, 0x01010101, 0) + __dp4a((int)o.y, 0x01010101, 0) + __dp4a((int)o.z, 0x01010101, 0) +
           __dp4a((int)o.w, 0x01010101, 0);
}

// block-wide sum of ints
__device__ __forceinline__ int block_sum_i32(int v, int* sm) {
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    int r = lane < ACT_THREADS / 32 ? sm[lane] : 0;
    for (int off = 16; off; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    __syncthreads();
    return r;
}

// block-wide max of non-negative floats (compared as bit patterns)
__device__ __forceinline__ float block_max_nonneg(float v, unsigned* sm) {
    unsigned u = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sm[warp] = u;
    __syncthreads();
    unsigned r = lane < ACT_THREADS / 32 ? sm[lane] : 0u;
    r = __reduce_max_sync(0xffffffffu, r);
    __syncthreads();
    return __uint_as_float(r);
}

__device__ __forceinline__ double block_sum_f64(double v, double* sm) {
    for (int off = 16; off; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) sm[warp] = v;
    __syncthreads();
    double r = lane < ACT_THREADS / 32 ? sm[lane] : 0.0;
    for (int off = 16; off; off >>= 1) r = __dadd_rn(r, __shfl_xor_sync(0xffffffffu, r, off));
    __syncthreads();
    return r;
}

// Quantise the n activations at xr (n % 16 == 0) with their own absmax:
// codes to qr, the floored absmax to *gamma_out and, when rowsum_out is not
// null, the sum of the codes to *rowsum_out.  Called by whole CTAs.
template <bool BF16>
__device__ __forceinline__ void quant_row(const char* xr, int n, int8_t* qr, float* gamma_out, unsigned* sm,
                                          int* rowsum_out = nullptr) {
    const int G = n / 16;
    float amax = 0.0f;
    for (int g = threadIdx.x; g < G; g += ACT_THREADS) {
        float v[16];
        load16<BF16>(xr, g, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
    amax = block_max_nonneg(amax, sm);
    const float gm = fmaxf(amax, 1e-5f);
    const float s = __fdiv_rn(127.0f, gm);
    int rs = 0;
    for (int g = threadIdx.x; g < G; g += ACT_THREADS) {
        float v[16];
        load16<BF16>(xr, g, v);
        rs += store16(qr, g, v, s);
    }
    if (rowsum_out) {  // uniform over the CTA
        rs = block_sum_i32(rs, reinterpret_cast<int*>(sm));
        if (threadIdx.x == 0) *rowsum_out = rs;
    }
    if (threadIdx.x == 0) *gamma_out = gm;
}

template <bool BF16>
__global__ void __launch_bounds__(ACT_THREADS) quant_act_kernel(const void* __restrict__ x, int K,
                                                                int8_t* __restrict__ x_q, float* __restrict__ gamma,
                                                                int* __restrict__ rowsum) {
    __shared__ unsigned sm[ACT_THREADS / 32];
    pdl_launch_dependents();
    pdl_wait();
    const long long row = blockIdx.x;
    const char* xr = reinterpret_cast<const char*>(x) + row * (long long)K * (BF16 ? 2 : 4);
    quant_row<BF16>(xr, K, x_q + row * (long long)K, gamma + row, sm, rowsum ? rowsum + row : nullptr);
}

// Group quantisation (unite.ai page, "Gruppenquantisierung und
// -normalisierung"): one CTA per (token m, channel group g) quantises
// x[m, g*Kg .. (g+1)*Kg) with its own absmax; codes go to the group-major
// x_q[g][m][:], the scale to gamma[m][g].
template <bool BF16>
__global__ void __launch_bounds__(ACT_THREADS) quant_act_grouped_kernel(const void* __restrict__ x, int K, int G,
                                                                        int M, int8_t* __restrict__ x_q,
                                                                        float* __restrict__ gamma) {
    __shared__ unsigned sm[ACT_THREADS / 32];
    pdl_launch_dependents();
    pdl_wait();
    const long long m = blockIdx.x / G;
    const int g = blockIdx.x % G;
    const int Kg = K / G;
    const char* xr = reinterpret_cast<const char*>(x) + (m * K + (long long)g * Kg) * (BF16 ? 2 : 4);
    quant_row<BF16>(xr, Kg, x_q + ((long long)g * M + m) * Kg, gamma + m * G + g, sm);
}

// h = combine(a, b) for 16 consecutive elements of group g.
__device__ __forceinline__ void combine16(const float* ar, const float* br, int combine, int g, float (&h)[16]) {
    const float4* pa = reinterpret_cast<const float4*>(ar) + 4 * g;
    const float4* pb = reinterpret_cast<const float4*>(br) + 4 * g;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 va = __ldg(pa + i);
        float av[4] = {va.x, va.y, va.z, va.w};
        if (combine == C_NONE) {
#pragma unroll
            for (int j = 0; j < 4; ++j) h[4 * i + j] = av[j];
        } else {
            float4 vb = __ldg(pb + i);
            float bv[4] = {vb.x, vb.y, vb.z, vb.w};
            if (combine == C_ADD) {
#pragma unroll
                for (int j = 0; j < 4; ++j) h[4 * i + j] = __fadd_rn(av[j], bv[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    double gd = (double)av[j];
                    double sg = __ddiv_rn(gd, __dadd_rn(1.0, exp(-gd)));
                    h[4 * i + j] = __double2float_rn(__dmul_rn(sg, (double)bv[j]));
                }
            }
        }
    }
}

// CACHE: the combined row h is kept in dynamic shared memory (K floats)
// between the two passes, so pass 2 neither re-reads a and b nor evaluates
// SiLU again; pass 1 (and so every reduction order) is the same either way.
template <bool CACHE>
__global__ void __launch_bounds__(ACT_THREADS) quant_act_rms_kernel(const float* __restrict__ a,
                                                                    const float* __restrict__ b, int combine, int K,
                                                                    float* __restrict__ h, int8_t* __restrict__ x_q,
                                                                    float* __restrict__ gamma) {
    __shared__ unsigned smu[ACT_THREADS / 32];
    __shared__ double smd[ACT_THREADS / 32];
    extern __shared__ float4 hcache[];  // K / 4 entries when CACHE
    pdl_launch_dependents();
    pdl_wait();
    const long long row = blockIdx.x;
    const float* ar = a + row * (long long)K;
    const float* br = b ? b + row * (long long)K : nullptr;
    float* hr = h ? h + row * (long long)K : nullptr;
    const int G = K / 16;
    float amax = 0.0f;
    double ss = 0.0;
    for (int g = threadIdx.x; g < G; g += ACT_THREADS) {
        float v[16];
        combine16(ar, br, combine, g, v);
        if (CACHE) {
#pragma unroll
            for (int i = 0; i < 4; ++i) hcache[4 * g + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        if (hr) {
            float4* ph = reinterpret_cast<float4*>(hr) + 4 * g;
#pragma unroll
            for (int i = 0; i < 4; ++i) ph[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = fmaxf(amax, fabsf(v[i]));
            ss = __dadd_rn(ss, __dmul_rn((double)v[i], (double)v[i]));
        }
    }
    if (!x_q) return;
    amax = block_max_nonneg(amax, smu);
    ss = block_sum_f64(ss, smd);
    const float gm = fmaxf(amax, 1e-5f);
    const float s = __fdiv_rn(127.0f, gm);
    const double ms = __dadd_rn(__ddiv_rn(ss, (double)K), 1e-6);
    const float rho = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(ms)));
    int8_t* qr = x_q + row * (long long)K;
    // (the block reductions above end in __syncthreads: the cache is complete)
    for (int g = threadIdx.x; g < G; g += ACT_THREADS) {
        float v[16];
        if (CACHE) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 c = hcache[4 * g + i];
                v[4 * i] = c.x;
                v[4 * i + 1] = c.y;
                v[4 * i + 2] = c.z;
                v[4 * i + 3] = c.w;
            }
        } else {
            combine16(ar, br, combine, g, v);
        }
        store16(qr, g, v, s);
    }
    if (threadIdx.x == 0) gamma[row] = __fmul_rn(rho, gm);
}

// ---- the RMS-folded quantiser over a thread-block cluster ----
//
// One row is shared by a cluster of RMS_CLUSTER CTAs, each taking a
// contiguous slice of its 16-element chunks, so that a long row (SiLU(gate) x
// up of a few thousand channels, with a binary64 exp per element) is not left
// to one CTA.  Every CTA forms h on its slice (kept in shared memory for pass
// 2), its max |h| and its binary64 sum of h^2 (per-thread strided partials,
// then the block trees); CTA 0 of the cluster reads the partials of all CTAs
// through distributed shared memory, adds the sums in rank order, and
// publishes 127 / gamma; every CTA then quantises its slice.
constexpr int RMS_CLUSTER = 8;
// a CTA's slice (40 KiB) and its static shared memory stay within the 48 KiB
// a launch may take without opting in
constexpr long long RMS_CLUSTER_MAX_K = 8LL * 40 * 1024 / 4;
// Measured: at M = 1 the cluster form saves ~1.5 us per call in the chained
// block and GLU; at M = 2048 it doubled the GLU's two quantiser passes.
constexpr long long RMS_CLUSTER_MAX_M = 64;

struct RmsPub {
    double ss;      // this CTA's sum of h^2
    unsigned amax;  // this CTA's max |h| (bit pattern)
    float s;        // (CTA 0) 127 / gamma of the row
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// All threads of all CTAs of the cluster; release / acquire at cluster scope.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of `p` (this CTA's shared memory) in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}

__device__ __forceinline__ double ld_cluster_f64(uint32_t a) {
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(a) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}

__global__ void __cluster_dims__(RMS_CLUSTER, 1, 1) __launch_bounds__(ACT_THREADS)
    quant_act_rms_cluster_kernel(const float* __restrict__ a, const float* __restrict__ b, int combine, int K,
                                 float* __restrict__ h, int8_t* __restrict__ x_q, float* __restrict__ gamma) {
    __shared__ unsigned smu[ACT_THREADS / 32];
    __shared__ double smd[ACT_THREADS / 32];
    __shared__ RmsPub pub;
    extern __shared__ float4 hcache[];  // this CTA's slice of h
    pdl_launch_dependents();
    pdl_wait();
    const long long row = blockIdx.y;
    const uint32_t rank = cluster_ctarank();
    const float* ar = a + row * (long long)K;
    const float* br = b ? b + row * (long long)K : nullptr;
    float* hr = h ? h + row * (long long)K : nullptr;
    const int G = K / 16;
    const int g0 = (int)((long long)G * rank / RMS_CLUSTER), g1 = (int)((long long)G * (rank + 1) / RMS_CLUSTER);
    float amax = 0.0f;
    double ss = 0.0;
    for (int g = g0 + (int)threadIdx.x; g < g1; g += ACT_THREADS) {
        float v[16];
        combine16(ar, br, combine, g, v);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            hcache[4 * (g - g0) + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        if (hr) {
            float4* ph = reinterpret_cast<float4*>(hr) + 4 * g;
#pragma unroll
            for (int i = 0; i < 4; ++i) ph[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            amax = fmaxf(amax, fabsf(v[i]));
            ss = __dadd_rn(ss, __dmul_rn((double)v[i], (double)v[i]));
        }
    }
    amax = block_max_nonneg(amax, smu);
    ss = block_sum_f64(ss, smd);
    if (threadIdx.x == 0) {
        pub.ss = ss;
        pub.amax = __float_as_uint(amax);
    }
    cluster_sync_all();  // every CTA's partials are visible to CTA 0
    if (rank == 0 && threadIdx.x == 0) {
        unsigned am = 0u;
        double tot = 0.0;
        for (uint32_t r = 0; r < RMS_CLUSTER; ++r) {
            tot = __dadd_rn(tot, ld_cluster_f64(cluster_addr(&pub.ss, r)));
            am = max(am, ld_cluster_u32(cluster_addr(&pub.amax, r)));
        }
        const float gm = fmaxf(__uint_as_float(am), 1e-5f);
        pub.s = __fdiv_rn(127.0f, gm);
        const double ms = __dadd_rn(__ddiv_rn(tot, (double)K), 1e-6);
        const float rho = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(ms)));
        if (x_q) gamma[row] = __fmul_rn(rho, gm);
    }
    cluster_sync_all();  // CTA 0's scale is visible to every CTA
    if (x_q) {
        const float s = __uint_as_float(ld_cluster_u32(cluster_addr(&pub.s, 0)));
        int8_t* qr = x_q + row * (long long)K;
        for (int g = g0 + (int)threadIdx.x; g < g1; g += ACT_THREADS) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 c = hcache[4 * (g - g0) + i];
                v[4 * i] = c.x;
                v[4 * i + 1] = c.y;
                v[4 * i + 2] = c.z;
                v[4 * i + 3] = c.w;
            }
            store16(qr, g, v, s);
        }
    }
    cluster_sync_all();  // no CTA leaves while another may still read its shared memory
}

}  // namespace

cudaError_t launch_quant_act(const void* x, bool bf16, long long M, long long K, int8_t* x_q, float* gamma,
                             cudaStream_t st, int* rowsum) {
    if (bf16)
        return launch_pdl(quant_act_kernel<true>, dim3((unsigned)M), dim3(ACT_THREADS), 0, st, x, (int)K, x_q, gamma,
                          rowsum);
    return launch_pdl(quant_act_kernel<false>, dim3((unsigned)M), dim3(ACT_THREADS), 0, st, x, (int)K, x_q, gamma,
                      rowsum);
}

cudaError_t launch_quant_act_grouped(const void* x, bool bf16, long long M, long long K, int G, int8_t* x_q,
                                     float* gamma, cudaStream_t st) {
    const dim3 grid((unsigned)(M * G));
    if (bf16)
        return launch_pdl(quant_act_grouped_kernel<true>, grid, dim3(ACT_THREADS), 0, st, x, (int)K, G, (int)M, x_q,
                          gamma);
    return launch_pdl(quant_act_grouped_kernel<false>, grid, dim3(ACT_THREADS), 0, st, x, (int)K, G, (int)M, x_q,
                      gamma);
}

cudaError_t launch_quant_act_rms(const float* a, const float* b, int combine, long long M, long long K, float* h,
                                 int8_t* x_q, float* gamma, cudaStream_t st) {
    if (K <= RMS_CLUSTER_MAX_K && M <= RMS_CLUSTER_MAX_M) {
        // few rows: one cluster of RMS_CLUSTER CTAs per row, each caching its
        // slice of h (many rows already fill the SMs with one CTA per row)
        const size_t slice = (size_t)((K / 16 + RMS_CLUSTER - 1) / RMS_CLUSTER) * 16 * 4;
        return launch_pdl(quant_act_rms_cluster_kernel, dim3(RMS_CLUSTER, (unsigned)M), dim3(ACT_THREADS), slice, st,
                          a, b, combine, (int)K, h, x_q, gamma);
    }
    // rows of up to 12288 channels (48 KiB, no opt-in needed) are cached between the passes
    constexpr long long CACHE_MAX_K = 48 * 1024 / 4;
    if (x_q && K <= CACHE_MAX_K)
        return launch_pdl(quant_act_rms_kernel<true>, dim3((unsigned)M), dim3(ACT_THREADS), (size_t)K * 4, st, a, b,
                          combine, (int)K, h, x_q, gamma);
    return launch_pdl(quant_act_rms_kernel<false>, dim3((unsigned)M), dim3(ACT_THREADS), 0, st, a, b, combine, (int)K,
                      h, x_q, gamma);
}

}  // namespace bl
