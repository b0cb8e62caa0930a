// k_gemv.cu -- decode BitLinear forward for M <= 64 tokens on CUDA cores.
//
// DataCamp blog "MatMul-free language models", section "MatMul vervangen
// door ternaire bewerkingen": with weights in {-1, 0, +1} every multiply is a
// negate, a zero or a pass-through, so the layer is a scaled ternary
// accumulation.  unite.ai page, eq. 3 "BitLinear-Betrieb": the integer result
// is rescaled by beta * gamma / Q_b.
//
// Design (HBM-bound at M = 1: the packed weights are > 99% of the bytes):
//   * one CTA per SM owns a contiguous slab of output rows, i.e. one
//     contiguous byte range of W_p; a producer warp streams it into a
//     shared-memory ring with 1-D bulk copies (cp.async.bulk, evict-first L2
//     hint), issuing every chunk that fits at kernel start so the whole
//     GPU's share of HBM requests is in flight from the first microsecond;
//     per-chunk mbarriers let compute start as soon as the first chunk lands;
//   * consumer "teams" of LPR lanes each take one row at a time; a lane
//     covers UPL 16-byte groups (64 trits each) of the row;
//   * the weight stream is requested before griddepcontrol.wait, so under
//     programmatic dependent launch it overlaps the activation quantiser;
//   * the contraction uses codes c = w + 1: sum_k c_k x_k - sum_k x_k =
//     sum_k w_k x_k.  A packed word holds the codes of k = 16j+4s+b at bits
//     8b+2s; masking with 0x03030303 << 2s (no shift) leaves 4^s * c in the
//     four bytes, so one LOP3 and one dp4a.u32.s32 per 4 trits accumulate
//     4^s * sum(c x) exactly in int32 (|partial| <= 4064 K < 2^31);
//   * team sums by warp shuffles; one lane writes y = (acc - rowsum) * f.
#include "common.cuh"
#include "kernels.cuh"

namespace bl {

namespace {

constexpr int GEMV_CWARPS = 8;                      // consumer warps
constexpr int GEMV_THREADS = (GEMV_CWARPS + 1) * 32;  // + 1 producer warp
constexpr int GEMV_MAX_STAGES = 32;
constexpr int GEMV_HDR = 2048;                      // barriers + per-token tables
constexpr int GEMV_MAX_M = 64;
constexpr int GEMV_RING_BYTES = 200 * 1024;
constexpr int GEMV_CHUNK_TARGET = 8192;

struct GemvParams {
    const int8_t* x_q;
    const float* gamma;
    const uint32_t* W_p;
    const float* beta;
    void* y;
    int M, K, N, mode;
    int rpc;           // packed rows per chunk
    int stages;        // ring depth
    int stage_stride;  // bytes per ring slot (multiple of 128)
};

struct Shared {
    uint64_t full[GEMV_MAX_STAGES];
    uint64_t empty[GEMV_MAX_STAGES];
    int abort_flag;
    int rowsum[GEMV_MAX_M];
    float fscale[GEMV_MAX_M];
};
static_assert(sizeof(Shared) <= GEMV_HDR, "header too large");

__device__ __forceinline__ void store_y(const GemvParams& p, int m, int n, int acc, float f) {
    const long long o = (long long)m * p.N + n;
    if (p.mode == Y_ACC) {
        reinterpret_cast<int*>(p.y)[o] = acc;
    } else {
        float v = __fmul_rn((float)acc, f);
        if (p.mode == Y_F32)
            reinterpret_cast<float*>(p.y)[o] = v;
        else
            reinterpret_cast<uint16_t*>(p.y)[o] = f32_to_bf16_rn(v);
    }
}

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

// Producer: stream this CTA's rows [r0, r0 + nrows) of W_p into the ring.
__device__ __forceinline__ void produce(const GemvParams& p, Shared& sh, unsigned char* ring, int r0, int nrows) {
    const int RB = p.K / 4;
    const int nchunks = (nrows + p.rpc - 1) / p.rpc;
    const uint64_t pol = policy_evict_first();
    const unsigned char* src = reinterpret_cast<const unsigned char*>(p.W_p) + (long long)r0 * RB;
    for (int c = 0; c < nchunks; ++c) {
        const int st = c % p.stages;
        if (c >= p.stages) {
            if (!mbar_wait(&sh.empty[st], ((c / p.stages) - 1) & 1)) {
                sh.abort_flag = 1;
                return;
            }
        }
        const int rows = min(p.rpc, nrows - c * p.rpc);
        const uint32_t bytes = (uint32_t)rows * RB;
        mbar_arrive_expect_tx(&sh.full[st], bytes);
        bulk_g2s(ring + (size_t)st * p.stage_stride, src + (long long)c * p.rpc * RB, bytes, &sh.full[st], pol);
    }
}

// Wait for the chunk holding slab row i; false once the CTA has aborted.
__device__ __forceinline__ bool wait_row(const GemvParams& p, Shared& sh, int i) {
    const int c = i / p.rpc;
    if (*(volatile int*)&sh.abort_flag) return false;
    if (!mbar_wait(&sh.full[c % p.stages], (c / p.stages) & 1)) {
        sh.abort_flag = 1;
        return false;
    }
    return true;
}

__device__ __forceinline__ void release_row(const GemvParams& p, Shared& sh, int i, int nchunks) {
    if (nchunks > p.stages) mbar_arrive(&sh.empty[(i / p.rpc) % p.stages]);
}

__device__ __forceinline__ void cta_rows(const GemvParams& p, int& r0, int& nrows) {
    const long long N = p.N;
    r0 = (int)((N * blockIdx.x) / gridDim.x);
    const int r1 = (int)((N * (blockIdx.x + 1)) / gridDim.x);
    nrows = r1 - r0;
}

__device__ __forceinline__ void init_barriers(const GemvParams& p, Shared& sh) {
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], p.rpc);
        }
        sh.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
}

// ---------------------------------------------------------------- M == 1

template <int LPR, int UPL>
__global__ void __launch_bounds__(GEMV_THREADS, 1) gemv_m1_kernel(const GemvParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Shared& sh = *reinterpret_cast<Shared*>(smem);
    unsigned char* ring = smem + GEMV_HDR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int r0, nrows;
    cta_rows(p, r0, nrows);
    init_barriers(p, sh);
    pdl_launch_dependents();
    if (warp == GEMV_CWARPS) {
        if (lane == 0) produce(p, sh, ring, r0, nrows);
        return;
    }
    pdl_wait();

    constexpr int T = GEMV_CWARPS * 32 / LPR;  // teams per CTA
    const int team = threadIdx.x / LPR;
    const int tl = lane % LPR;
    const int K4 = p.K / 64;                   // 16-byte groups per row
    const int RB = p.K / 4;
    const int nchunks = (nrows + p.rpc - 1) / p.rpc;

    int xr[UPL][16];
    int rs = 0;
#pragma unroll
    for (int u = 0; u < UPL; ++u) {
        const int idx = tl + u * LPR;
        if (idx < K4) {
            const int4* px = reinterpret_cast<const int4*>(p.x_q) + 4 * idx;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                int4 v = __ldg(px + q);
                xr[u][4 * q + 0] = v.x;
                xr[u][4 * q + 1] = v.y;
                xr[u][4 * q + 2] = v.z;
                xr[u][4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) xr[u][q] = 0;
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) rs += bytesum_s8(xr[u][q]);
    }
#pragma unroll
    for (int off = LPR / 2; off; off >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, off);
    // beta and gamma are absent (NULL) when only the accumulators are wanted
    const float f = p.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(__ldg(p.beta), __ldg(p.gamma)), 127.0f);

    // Warp-uniform trip count: every lane runs every shuffle.
    const int iters = (nrows + T - 1) / T;
    for (int it = 0; it < iters; ++it) {
        const int i = it * T + team;
        const bool valid = i < nrows;
        bool ok = valid && wait_row(p, sh, i);
        int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
        if (ok) {
            const int c = i / p.rpc;
            const uint4* wrow = reinterpret_cast<const uint4*>(ring + (size_t)(c % p.stages) * p.stage_stride +
                                                                (size_t)(i - c * p.rpc) * RB);
#pragma unroll
            for (int u = 0; u < UPL; ++u) {
                const int idx = tl + u * LPR;
                if (idx < K4) {
                    const uint4 w = wrow[idx];
                    word_dot(w.x, xr[u][0], xr[u][1], xr[u][2], xr[u][3], a0, a1, a2, a3);
                    word_dot(w.y, xr[u][4], xr[u][5], xr[u][6], xr[u][7], a0, a1, a2, a3);
                    word_dot(w.z, xr[u][8], xr[u][9], xr[u][10], xr[u][11], a0, a1, a2, a3);
                    word_dot(w.w, xr[u][12], xr[u][13], xr[u][14], xr[u][15], a0, a1, a2, a3);
                }
            }
        }
        int acc = combine4(a0, a1, a2, a3);
#pragma unroll
        for (int off = LPR / 2; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (ok && tl == 0) {
            release_row(p, sh, i, nchunks);
            store_y(p, 0, r0 + i, acc - rs, f);
        }
    }
}

// ------------------------------------------------------------ 1 < M <= 64

template <int MT>
__global__ void __launch_bounds__(GEMV_THREADS, 1) gemv_mt_kernel(const GemvParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Shared& sh = *reinterpret_cast<Shared*>(smem);
    unsigned char* ring = smem + GEMV_HDR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int r0, nrows;
    cta_rows(p, r0, nrows);
    init_barriers(p, sh);
    pdl_launch_dependents();
    if (warp == GEMV_CWARPS) {
        if (lane == 0) produce(p, sh, ring, r0, nrows);
        return;
    }
    pdl_wait();

    const int K4 = p.K / 64;
    const int RB = p.K / 4;
    const int nchunks = (nrows + p.rpc - 1) / p.rpc;
    // per-token row sums of x_q and rescale factors
    for (int m = warp; m < p.M; m += GEMV_CWARPS) {
        const int4* px = reinterpret_cast<const int4*>(p.x_q + (long long)m * p.K);
        int s = 0;
        for (int g = lane; g < p.K / 16; g += 32) {
            int4 v = __ldg(px + g);
            s += bytesum_s8(v.x) + bytesum_s8(v.y) + bytesum_s8(v.z) + bytesum_s8(v.w);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            sh.rowsum[m] = s;
            sh.fscale[m] = p.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(__ldg(p.beta), __ldg(p.gamma + m)), 127.0f);
        }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(GEMV_CWARPS * 32) : "memory");

    for (int i = warp; i < nrows; i += GEMV_CWARPS) {
        // every lane waits the same barrier; the decision is made warp-uniform
        if (!__all_sync(0xffffffffu, wait_row(p, sh, i))) break;
        const int c = i / p.rpc;
        const uint4* wrow = reinterpret_cast<const uint4*>(ring + (size_t)(c % p.stages) * p.stage_stride +
                                                            (size_t)(i - c * p.rpc) * RB);
        for (int m0 = 0; m0 < p.M; m0 += MT) {
            int a[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m) a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0;
            for (int idx = lane; idx < K4; idx += 32) {
                const uint4 w = wrow[idx];
                const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m0 + m < p.M) {
                        const int4* px = reinterpret_cast<const int4*>(p.x_q + (long long)(m0 + m) * p.K) + 4 * idx;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int4 xv = __ldg(px + q);
                            word_dot(wv[q], xv.x, xv.y, xv.z, xv.w, a[m][0], a[m][1], a[m][2], a[m][3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                int acc = combine4(a[m][0], a[m][1], a[m][2], a[m][3]);
#pragma unroll
                for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (lane == 0 && m0 + m < p.M) store_y(p, m0 + m, r0 + i, acc - sh.rowsum[m0 + m], sh.fscale[m0 + m]);
            }
        }
        __syncwarp();
        if (lane == 0) release_row(p, sh, i, nchunks);
    }
}

// ------------------------------------------------------------------- host

template <typename K>
cudaError_t launch_with_smem(K kernel, int grid, size_t smem, cudaStream_t st, const GemvParams& p) {
    cudaError_t e = ensure_smem_optin(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, dim3(grid), dim3(GEMV_THREADS), smem, st, p);
}

using M1Kernel = void (*)(const GemvParams);

template <int LPR>
M1Kernel m1_kernel_for(int upl) {
    switch (upl) {
        case 1: return gemv_m1_kernel<LPR, 1>;
        case 2: return gemv_m1_kernel<LPR, 2>;
        case 3: return gemv_m1_kernel<LPR, 3>;
        case 4: return gemv_m1_kernel<LPR, 4>;
        case 5: return gemv_m1_kernel<LPR, 5>;
        case 6: return gemv_m1_kernel<LPR, 6>;
        case 7: return gemv_m1_kernel<LPR, 7>;
        case 8: return gemv_m1_kernel<LPR, 8>;
    }
    return nullptr;
}

}  // namespace

cudaError_t launch_gemv(const int8_t* x_q, const float* gamma, int M, int K, const uint32_t* W_p, const float* beta,
                        int N, void* y, YMode mode, const DevInfo& dev, cudaStream_t st) {
    GemvParams p;
    p.x_q = x_q;
    p.gamma = gamma;
    p.W_p = W_p;
    p.beta = beta;
    p.y = y;
    p.M = M;
    p.K = K;
    p.N = N;
    p.mode = mode;
    const int RB = K / 4;
    const int grid = std::max(1, std::min(N, dev.num_sms));
    const int rows_per_cta = (N + grid - 1) / grid;
    p.rpc = std::max(1, std::min(rows_per_cta, GEMV_CHUNK_TARGET / RB));
    p.stage_stride = ((p.rpc * RB) + 127) / 128 * 128;
    const int nchunks = (rows_per_cta + p.rpc - 1) / p.rpc;
    const int max_ring = std::min(GEMV_RING_BYTES, dev.max_smem_optin - GEMV_HDR);
    p.stages = std::max(1, std::min({max_ring / p.stage_stride, GEMV_MAX_STAGES, nchunks}));
    const size_t smem = GEMV_HDR + (size_t)p.stages * p.stage_stride;

    const int K4 = K / 64;
    if (M == 1 && K4 <= 8 * 32) {
        // pick lanes-per-row and groups-per-lane to cover K4 with least idle lanes
        int best_lpr = 32, best_upl = (K4 + 31) / 32;
        double best_eff = -1.0;
        for (int lpr : {32, 16, 8}) {
            const int upl = (K4 + lpr - 1) / lpr;
            if (upl > 8) continue;
            const double eff = (double)K4 / (lpr * upl);
            if (eff > best_eff + 1e-9) {
                best_eff = eff;
                best_lpr = lpr;
                best_upl = upl;
            }
        }
        M1Kernel k = best_lpr == 32 ? m1_kernel_for<32>(best_upl)
                     : best_lpr == 16 ? m1_kernel_for<16>(best_upl)
                                      : m1_kernel_for<8>(best_upl);
        return launch_with_smem(k, grid, smem, st, p);
    }
    if (M <= 1) return launch_with_smem(gemv_mt_kernel<1>, grid, smem, st, p);
    if (M <= 2) return launch_with_smem(gemv_mt_kernel<2>, grid, smem, st, p);
    if (M <= 4) return launch_with_smem(gemv_mt_kernel<4>, grid, smem, st, p);
    return launch_with_smem(gemv_mt_kernel<8>, grid, smem, st, p);
}

}  // namespace bl
