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
//     hint), issuing every chunk that fits as soon as the CTA starts, so the
//     GPU's whole share of HBM requests is in flight from the first
//     microsecond and the stream overlaps the previous kernel's tail under
//     programmatic dependent launch;
//   * the contraction uses codes c = w + 1: sum_k c_k x_k - sum_k x_k =
//     sum_k w_k x_k.  A packed word holds the codes of k = 16j+4s+b at bits
//     8b+2s; masking with 0x03030303 << 2s (no shift) leaves 4^s * c in the
//     four bytes, so one LOP3 and one dp4a.u32.s32 per 4 trits accumulate
//     4^s * sum(c x) exactly in int32 (|partial| <= 4064 K < 2^31);
//   * M <= 4 ("small" kernel): the activations live in shared memory (with an
//     XOR swizzle of the 16-byte chunks that makes the per-lane reads
//     bank-conflict free); a team of LPR lanes works on R rows at once so
//     every lane keeps 4 * R * MT independent dp4a chains in flight, and the
//     R * MT team sums are finished by one batched transpose-reduction of
//     warp shuffles.  The quantiser can run in the prologue (fused forward),
//     so a decode layer is a single kernel;
//   * 4 < M <= 64 ("mt" kernel): one warp per row, activations read through
//     L1 from global memory, MT tokens per pass.
#include "act_inl.cuh"
#include "common.cuh"
#include "gemv_inl.cuh"
#include "kernels.cuh"

namespace bl {

namespace {

constexpr int GEMV_MAX_STAGES = 32;
constexpr int GEMV_HDR = 4096;  // barriers + per-token tables + reduction scratch
constexpr int GEMV_MAX_M = 64;
constexpr int GEMV_MAX_CWARPS = 13;                           // small kernel: <= 448 threads and
constexpr int GEMV_MAX_THREADS = (GEMV_MAX_CWARPS + 1) * 32;  // <= 73 registers: two CTAs fit an SM
constexpr int GEMV_KS_MAX_ROWS = 64;                          // rows per CTA when K is split
constexpr int GEMV_CO_RESIDENT = 2;                           // a kernel and its PDL successor
constexpr int GEMV_MT_CWARPS = 8;  // consumer warps of the mt kernel
constexpr int GEMV_CHUNK_TARGET = 8192;
constexpr int GEMV_XQ_SMEM_MAX = 64 * 1024;
constexpr int GEMV_SMALL_MAX_M = 4;
constexpr int GEMV_EARLY_CHUNKS = 2;  // chunks issued before the CTA barrier

struct GemvParams {
    const void* x;  // fp32/bf16 activations when the quantiser is fused
    const int8_t* x_q;
    const float* gamma;
    const uint32_t* W_p;
    const float* beta;
    void* y;
    int M, K, N, mode, x_mode;
    int rb;            // bytes per packed weight row: K / 4 (2-bit trits) or K / 8 (1-bit signs)
    int rpc;           // packed rows per chunk (a power of two)
    int rpc_shift;     // log2(rpc)
    int reuse;         // 0: every chunk has its own ring slot (slot = chunk, parity 0)
    int stages;        // ring depth
    int stage_stride;  // bytes per ring slot (rpc rows, a multiple of 16)
    int xq_bytes;      // shared-memory bytes reserved for x_q (small kernel)
    int ks;            // K slices per row (small kernel): 1, 2 or 4
    int slice4;        // 16-byte weight groups per slice
    int wave;          // mt kernel: rows in flight per wave
    long long wait_limit;  // small kernel: SM cycles before a wait gives up
    int stall_cta;         // small kernel test hook: this CTA's producer issues nothing (-1: none)
};

struct Shared {
    uint64_t full[GEMV_MAX_STAGES];
    uint64_t empty[GEMV_MAX_STAGES];
    int abort_flag;
    float beta;  // read at CTA start (a weight input, like W_p)
    int rowsum[GEMV_MAX_M];
    float fscale[GEMV_MAX_M];
    unsigned red_u[GEMV_MAX_CWARPS][GEMV_SMALL_MAX_M];
    int red_i[GEMV_MAX_CWARPS][GEMV_SMALL_MAX_M];
    int part[GEMV_KS_MAX_ROWS][GEMV_SMALL_MAX_M];  // K-slice partial sums
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

// 1-bit weights (unite.ai page, "Gewichtsbinarisierung"): the sign of
// k = 32j + 4s + b is bit 8b + s of word j (set for +1).  Masking with
// 0x01010101 << s leaves 2^s * bit in the four bytes; the upper half
// (s = 4..7) is brought down by one shift of the word, so four chains of
// 2^s * sum(bit * x) cover the 32 weights.  x0 holds x of k = 32j .. 32j+15
// (int s = k 4s .. 4s+3) and x1 of k = 32j+16 .. 32j+31.
__device__ __forceinline__ void bits_dot(uint32_t w, const int4& x0, const int4& x1, int& a0, int& a1, int& a2,
                                         int& a3) {
    a0 = dp4a_us(w & 0x01010101u, x0.x, a0);
    a1 = dp4a_us(w & 0x02020202u, x0.y, a1);
    a2 = dp4a_us(w & 0x04040404u, x0.z, a2);
    a3 = dp4a_us(w & 0x08080808u, x0.w, a3);
    const uint32_t h = w >> 4;
    a0 = dp4a_us(h & 0x01010101u, x1.x, a0);
    a1 = dp4a_us(h & 0x02020202u, x1.y, a1);
    a2 = dp4a_us(h & 0x04040404u, x1.z, a2);
    a3 = dp4a_us(h & 0x08080808u, x1.w, a3);
}

__device__ __forceinline__ int combine_bits(int a0, int a1, int a2, int a3) {
    return a0 + (a1 >> 1) + (a2 >> 2) + (a3 >> 3);  // each a_s is a multiple of 2^s
}

// Row result from the contraction with the stored codes: ternary codes
// c = w + 1 give sum c x - sum x; sign bits give 2 sum bit x - sum x.
template <int WB>
__device__ __forceinline__ int finish_acc(int dot, int rowsum) {
    return WB == 2 ? dot - rowsum : 2 * dot - rowsum;
}

// Ring slot and phase parity of chunk c.  Without reuse the whole slab fits
// (slot = c, first phase); otherwise slots cycle through the ring.
__device__ __forceinline__ int chunk_slot(const GemvParams& p, int c) { return p.reuse ? c % p.stages : c; }
__device__ __forceinline__ uint32_t chunk_parity(const GemvParams& p, int c) {
    return p.reuse ? (uint32_t)((c / p.stages) & 1) : 0u;
}

// Producer: stream chunks [c0, c1) of this CTA's rows [r0, r0 + nrows) of W_p
// into the ring (a chunk is rpc rows; chunk c goes to slot c % stages).
__device__ __forceinline__ void produce(const GemvParams& p, Shared& sh, unsigned char* ring, int r0, int nrows,
                                        int c0, int c1) {
    const int RB = p.rb;
    const uint64_t pol = policy_evict_first();
    const unsigned char* src = reinterpret_cast<const unsigned char*>(p.W_p) + (long long)r0 * RB;
    for (int c = c0; c < c1; ++c) {
        const int st = chunk_slot(p, c);
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

// Wait (at most `limit` SM cycles) for the phase of the given parity; false,
// with the device error word raised, if it did not complete in time.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) {
            set_dev_error(DEV_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Wait for the chunk holding slab row i; false once the CTA has aborted.
__device__ __forceinline__ bool wait_row(const GemvParams& p, Shared& sh, int i) {
    const int c = i >> p.rpc_shift;
    if (*(volatile int*)&sh.abort_flag) return false;
    if (!mbar_wait_limit(&sh.full[chunk_slot(p, c)], chunk_parity(p, c), p.wait_limit)) {
        sh.abort_flag = 1;
        return false;
    }
    return true;
}

__device__ __forceinline__ void release_row(const GemvParams& p, Shared& sh, int i) {
    if (p.reuse) mbar_arrive(&sh.empty[chunk_slot(p, i >> p.rpc_shift)]);
}

__device__ __forceinline__ const uint4* row_ptr(const GemvParams& p, const unsigned char* ring, int i) {
    const int c = i >> p.rpc_shift;
    return reinterpret_cast<const uint4*>(ring + (size_t)chunk_slot(p, c) * p.stage_stride +
                                          (size_t)(i & (p.rpc - 1)) * p.rb);
}

__device__ __forceinline__ void cta_rows(const GemvParams& p, int cta, int ncta, int& r0, int& nrows) {
    const long long N = p.N;
    r0 = (int)((N * cta) / ncta);
    const int r1 = (int)((N * (cta + 1)) / ncta);
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

__device__ __forceinline__ void consumer_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// 16-byte chunk c of a token's x_q row is stored at slot c ^ ((c >> 3) & 3)
// for 2-bit weights, where lane l of a team reads chunks 4l + q, and at slot
// c ^ ((c >> 3) & 7) for 1-bit weights, where it reads chunks 8l + q: either
// way the eight lanes of one shared-memory phase hit distinct bank groups.
template <int WB>
__device__ __forceinline__ int xq_slot(int c) { return c ^ ((c >> 3) & (WB == 2 ? 3 : 7)); }

// Fill the shared x_q rows (tokens 0..MT-1; tokens >= M are zero), rowsum[]
// and fscale[].  Runs on the consumer threads only.  The first XC chunks per
// token of every thread are loaded at once into registers and serve both the
// absmax pass and the quantisation pass, so the stage costs one memory round
// trip (x was just written by the preceding kernel and sits in L2).
template <int MT, int XM, int WB>
__device__ __forceinline__ void stage_activations(const GemvParams& p, Shared& sh, int4* xsm, int ctid, int cthreads,
                                                  int cwarps) {
    const int G = p.K / 16;  // 16-byte chunks per token
    const int lane = ctid & 31, warp = ctid >> 5;
    constexpr int XC = XM == X_F32 ? (MT <= 2 ? 2 / MT : 0) : 4 / MT;  // <= 32 registers of cache
    constexpr int XCA = XC > 0 ? XC : 1;
    constexpr int TB = XM == X_F32 ? (MT < 2 ? MT : 2) : MT;            // tokens loaded together past the cache
    const size_t xrow = (size_t)p.K * (XM == X_BF16 ? 2 : XM == X_F32 ? 4 : 1);
    const char* xbase = XM == X_QUANTISED ? reinterpret_cast<const char*>(p.x_q) : reinterpret_cast<const char*>(p.x);
    XChunk<XM> cache[MT][XCA];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int i = 0; i < XC; ++i) {
            const int g = ctid + i * cthreads;
            if (m < p.M && g < G) ld_chunk<XM>(xbase + (size_t)m * xrow, g, cache[m][i]);
        }
    }
    float s[MT];
    float gam[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) s[m] = gam[m] = 0.0f;
    if (XM != X_QUANTISED) {
        // pass 1: per-token absmax over the row (exact, order-free); chunks
        // beyond the cache are loaded TB tokens at a time, so that their
        // loads are in flight together
        unsigned amax[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            amax[m] = 0u;
#pragma unroll
            for (int i = 0; i < XC; ++i)
                if (m < p.M && ctid + i * cthreads < G) amax[m] = chunk_absmax<XM>(cache[m][i], amax[m]);
        }
#pragma unroll
        for (int m0 = 0; m0 < MT; m0 += TB) {
            for (int g = ctid + XC * cthreads; g < G; g += cthreads) {
                XChunk<XM> c[TB];
#pragma unroll
                for (int t = 0; t < TB; ++t)
                    if (m0 + t < p.M) ld_chunk<XM>(xbase + (size_t)(m0 + t) * xrow, g, c[t]);
#pragma unroll
                for (int t = 0; t < TB; ++t)
                    if (m0 + t < p.M) amax[m0 + t] = chunk_absmax<XM>(c[t], amax[m0 + t]);
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const unsigned a = __reduce_max_sync(0xffffffffu, amax[m]);
            if (lane == 0) sh.red_u[warp][m] = a;
        }
        consumer_sync(cthreads);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            unsigned a = 0u;
            for (int w = 0; w < cwarps; ++w) a = max(a, sh.red_u[w][m]);
            gam[m] = fmaxf(__uint_as_float(a), 1e-5f);
            s[m] = __fdiv_rn(127.0f, gam[m]);
        }
        if (ctid < MT) {
            float f = 0.0f;
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m == ctid && p.mode != Y_ACC && m < p.M) f = __fdiv_rn(__fmul_rn(sh.beta, gam[m]), 127.0f);
            sh.fscale[ctid] = f;
        }
    } else if (ctid < MT) {
        const int m = ctid;
        sh.fscale[m] = p.mode != Y_ACC && m < p.M ? __fdiv_rn(__fmul_rn(sh.beta, __ldg(p.gamma + m)), 127.0f) : 0.0f;
    }
    for (int i = ctid; i < GEMV_KS_MAX_ROWS * GEMV_SMALL_MAX_M; i += cthreads) (&sh.part[0][0])[i] = 0;
    // pass 2: write x_q chunks into their swizzled slots, accumulate row sums
    int rs[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        rs[m] = 0;
        int4* dst = xsm + (size_t)m * G;
#pragma unroll
        for (int i = 0; i < XC; ++i) {
            const int g = ctid + i * cthreads;
            if (g < G) {
                int4 q = make_int4(0, 0, 0, 0);
                if (m < p.M) {
                    q = chunk_codes<XM>(cache[m][i], s[m]);
                    rs[m] += bytesum_s8(q.x) + bytesum_s8(q.y) + bytesum_s8(q.z) + bytesum_s8(q.w);
                }
                dst[xq_slot<WB>(g)] = q;
            }
        }
    }
#pragma unroll
    for (int m0 = 0; m0 < MT; m0 += TB) {
        for (int g = ctid + XC * cthreads; g < G; g += cthreads) {
            XChunk<XM> c[TB];
#pragma unroll
            for (int t = 0; t < TB; ++t)
                if (m0 + t < p.M) ld_chunk<XM>(xbase + (size_t)(m0 + t) * xrow, g, c[t]);
#pragma unroll
            for (int t = 0; t < TB; ++t) {
                const int m = m0 + t;
                int4 q = make_int4(0, 0, 0, 0);
                if (m < p.M) {
                    q = chunk_codes<XM>(c[t], s[m]);
                    rs[m] += bytesum_s8(q.x) + bytesum_s8(q.y) + bytesum_s8(q.z) + bytesum_s8(q.w);
                }
                xsm[(size_t)m * G + xq_slot<WB>(g)] = q;
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        int v = rs[m];
#pragma unroll
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0 && v != 0) atomicAdd(&sh.rowsum[m], v);
    }
    consumer_sync(cthreads);
}

// ---------------------------------------------------------------- M <= 4

// One CTA's share (CTA `cta` of `ncta` working on problem p) of the M <= 4 forward.
template <int LPR, int MT, int R, int XM, int WB>
__device__ __forceinline__ void gemv_small_body(const GemvParams& p, int cta, int ncta, unsigned char* smem) {
    Shared& sh = *reinterpret_cast<Shared*>(smem);
    int4* xsm = reinterpret_cast<int4*>(smem + GEMV_HDR);
    unsigned char* ring = smem + GEMV_HDR + p.xq_bytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cwarps = blockDim.x / 32 - 1;  // warp 0 produces, warps 1.. consume
    const int cthreads = cwarps * 32;
    int r0, nrows;
    cta_rows(p, cta, ncta, r0, nrows);
    const int nchunks = (nrows + p.rpc - 1) / p.rpc;
    // Thread 0 sets up the barriers and puts the first chunks in flight before
    // anyone else runs, so the HBM stream starts at once; the producer warp
    // issues the rest after the CTA barrier.  (Issuing the whole slab here
    // stalled the CTA barrier -- and so the consumers -- for microseconds when
    // the memory system pushed back.)
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], p.rpc * p.ks);  // every K slice of every row releases once
        }
        sh.abort_flag = 0;
        for (int m = 0; m < GEMV_SMALL_MAX_M; ++m) sh.rowsum[m] = 0;
        // beta and W_p are weight inputs, not written by the preceding kernel:
        // read before waiting for it
        sh.beta = p.mode == Y_ACC ? 0.0f : __ldg(p.beta);
        fence_mbar_init();
        if (cta != p.stall_cta) produce(p, sh, ring, r0, nrows, 0, min(nchunks, GEMV_EARLY_CHUNKS));
    }
    __syncthreads();
    pdl_launch_dependents();
    if (warp == 0) {
        if (lane == 0 && nchunks > GEMV_EARLY_CHUNKS && cta != p.stall_cta)
            produce(p, sh, ring, r0, nrows, GEMV_EARLY_CHUNKS, nchunks);
        return;
    }
    pdl_wait();
    const int ctid = threadIdx.x - 32;
    stage_activations<MT, XM, WB>(p, sh, xsm, ctid, cthreads, cwarps);

    constexpr int V = R * MT;
    const int T = cthreads / LPR;  // teams
    const int team = ctid / LPR;
    const int tl = ctid % LPR;
    const int K4 = p.rb / 16;  // 16-byte groups of packed weights per row
    const int G = p.K / 16;    // 16-byte chunks of x_q per token
    const int KS = p.ks;
    // work item = (group of R rows, K slice); warp-uniform trip count
    const int items = (nrows + R - 1) / R * KS;
    const int iters = (items + T - 1) / T;

    for (int it = 0; it < iters; ++it) {
        const int item = it * T + team;
        const int b = (item / KS) * R;
        const int sl = item % KS;
        const int k_lo = sl * p.slice4, k_hi = min(K4, k_lo + p.slice4);
        const int nvalid = item < items ? max(0, min(R, nrows - b)) : 0;
        bool ok = nvalid > 0;
        for (int r = 0; r < nvalid; ++r) ok = ok && wait_row(p, sh, b + r);
        // row offsets once per team-iteration (missing rows alias row b)
        uint32_t ro[R];
#pragma unroll
        for (int r = 0; r < R; ++r)
            ro[r] = ok ? (uint32_t)(reinterpret_cast<const unsigned char*>(row_ptr(p, ring, b + (r < nvalid ? r : 0))) -
                                    ring)
                       : 0u;
        int a[R][MT][4];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) a[r][m][0] = a[r][m][1] = a[r][m][2] = a[r][m][3] = 0;
        if (ok && k_lo + tl < k_hi) {
            // software pipeline: the next group's weights load while this one is used
            uint4 wn[R];
#pragma unroll
            for (int r = 0; r < R; ++r) wn[r] = *reinterpret_cast<const uint4*>(ring + ro[r] + 16 * (k_lo + tl));
            for (int idx = k_lo + tl; idx < k_hi; idx += LPR) {
                uint4 w[R];
#pragma unroll
                for (int r = 0; r < R; ++r) w[r] = wn[r];
                const int nxt = idx + LPR < k_hi ? idx + LPR : idx;
#pragma unroll
                for (int r = 0; r < R; ++r) wn[r] = *reinterpret_cast<const uint4*>(ring + ro[r] + 16 * nxt);
                if constexpr (WB == 2) {
                    const int key = (idx >> 1) & 3;  // swizzle of chunks 4 idx .. 4 idx + 3
                    const int4* xb = xsm + 4 * idx;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            const int4 xv = xb[m * G + (q ^ key)];
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const uint32_t wq = q == 0 ? w[r].x : q == 1 ? w[r].y : q == 2 ? w[r].z : w[r].w;
                                word_dot(wq, xv.x, xv.y, xv.z, xv.w, a[r][m][0], a[r][m][1], a[r][m][2],
                                         a[r][m][3]);
                            }
                        }
                    }
                } else {
                    const int key = idx & 7;  // swizzle of chunks 8 idx .. 8 idx + 7
                    const int4* xb = xsm + 8 * idx;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            const int4 x0 = xb[m * G + ((2 * q) ^ key)];
                            const int4 x1 = xb[m * G + ((2 * q + 1) ^ key)];
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const uint32_t wq = q == 0 ? w[r].x : q == 1 ? w[r].y : q == 2 ? w[r].z : w[r].w;
                                bits_dot(wq, x0, x1, a[r][m][0], a[r][m][1], a[r][m][2], a[r][m][3]);
                            }
                        }
                    }
                }
            }
        }
        int vals[V];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m)
                vals[r * MT + m] = WB == 2 ? combine4(a[r][m][0], a[r][m][1], a[r][m][2], a[r][m][3])
                                           : combine_bits(a[r][m][0], a[r][m][1], a[r][m][2], a[r][m][3]);
        int which;
        const int tot = team_reduce<LPR, V>(vals, tl, which);
        // lane tl = which * (LPR / V) is the first lane that owns value `which`
        if (ok && tl == which * (LPR / V)) {
            const int r = which / MT, m = which % MT;
            if (r < nvalid) {
                if (m == 0) release_row(p, sh, b + r);
                if (KS == 1) {
                    if (m < p.M) store_y(p, m, r0 + b + r, finish_acc<WB>(tot, sh.rowsum[m]), sh.fscale[m]);
                } else {
                    atomicAdd(&sh.part[b + r][m], tot);
                }
            }
        }
        // With a recycled ring, the rows of one iteration fit strictly inside
        // the ring (host-side sizing) and no team starts the next iteration
        // before all have finished this one: a parity wait then never meets a
        // slot two loads behind the one it asks for.
        if (p.reuse) consumer_sync(cthreads);
    }
    if (KS > 1) {  // all slices of every row are in: finish the rows
        consumer_sync(cthreads);
        for (int i = ctid; i < nrows * MT; i += cthreads) {
            const int r = i / MT, m = i % MT;
            if (m < p.M) store_y(p, m, r0 + r, finish_acc<WB>(sh.part[r][m], sh.rowsum[m]), sh.fscale[m]);
        }
    }
}

template <int LPR, int MT, int R, int XM, int WB>
__global__ void __launch_bounds__(GEMV_MAX_THREADS, GEMV_CO_RESIDENT) gemv_small_kernel(const GemvParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    gemv_small_body<LPR, MT, R, XM, WB>(p, blockIdx.x, gridDim.x, smem);
}

// Several independent problems (same M, same x / y formats) in one launch:
// CTAs [cta0[i], cta0[i+1]) work on problem i.  Each problem keeps its own
// launch shape (lanes per row); the block size is the largest of them.
constexpr int GEMV_GROUP_MAX = 8;

struct GroupParams {
    GemvParams prob[GEMV_GROUP_MAX];
    int lpr[GEMV_GROUP_MAX];
    int cta0[GEMV_GROUP_MAX + 1];
    int count;
};

template <int MT, int R, int XM>
__global__ void __launch_bounds__(GEMV_MAX_THREADS, GEMV_CO_RESIDENT) gemv_group_kernel(const __grid_constant__ GroupParams g) {
    extern __shared__ __align__(128) unsigned char smem[];
    int i = 0;
    while (i + 1 < g.count && (int)blockIdx.x >= g.cta0[i + 1]) ++i;
    const int cta = blockIdx.x - g.cta0[i], ncta = g.cta0[i + 1] - g.cta0[i];
    if (g.lpr[i] == 32)
        gemv_small_body<32, MT, R, XM, 2>(g.prob[i], cta, ncta, smem);
    else if (g.lpr[i] == 16)
        gemv_small_body<16, MT, R, XM, 2>(g.prob[i], cta, ncta, smem);
    else
        gemv_small_body<8, MT, R, XM, 2>(g.prob[i], cta, ncta, smem);
}

// ------------------------------------------------------------ 4 < M <= 64

template <int MT>
__global__ void __launch_bounds__((GEMV_MT_CWARPS + 1) * 32, 1) gemv_mt_kernel(const GemvParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    Shared& sh = *reinterpret_cast<Shared*>(smem);
    unsigned char* ring = smem + GEMV_HDR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int r0, nrows;
    cta_rows(p, blockIdx.x, gridDim.x, r0, nrows);
    init_barriers(p, sh);
    pdl_launch_dependents();
    if (warp == GEMV_MT_CWARPS) {
        if (lane == 0) produce(p, sh, ring, r0, nrows, 0, (nrows + p.rpc - 1) / p.rpc);
        return;
    }
    pdl_wait();

    const int K4 = p.K / 64;
    const int nchunks = (nrows + p.rpc - 1) / p.rpc;
    // per-token row sums of x_q and rescale factors
    for (int m = warp; m < p.M; m += GEMV_MT_CWARPS) {
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
            // beta and gamma are absent (NULL) when only the accumulators are wanted
            sh.fscale[m] = p.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(__ldg(p.beta), __ldg(p.gamma + m)), 127.0f);
        }
    }
    consumer_sync(GEMV_MT_CWARPS * 32);

    // rows go out in waves of p.wave (<= consumer warps); with a recycled ring a
    // wave fits strictly inside it and waves are separated by a barrier
    for (int base = 0; base < nrows; base += p.wave) {
        const int i = base + warp;
        const bool mine = warp < p.wave && i < nrows;
        // every lane waits the same barrier; the decision is made warp-uniform
        const bool ok = __all_sync(0xffffffffu, mine && wait_row(p, sh, i));
        if (ok) {
            const uint4* wrow = row_ptr(p, ring, i);
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
                            const int4* px =
                                reinterpret_cast<const int4*>(p.x_q + (long long)(m0 + m) * p.K) + 4 * idx;
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
                    if (lane == 0 && m0 + m < p.M)
                        store_y(p, m0 + m, r0 + i, acc - sh.rowsum[m0 + m], sh.fscale[m0 + m]);
                }
            }
            __syncwarp();
            if (lane == 0) release_row(p, sh, i);
        }
        if (p.reuse) consumer_sync(GEMV_MT_CWARPS * 32);
    }
}

// ------------------------------------------------------------------- host

template <typename KernelT>
cudaError_t launch_with_smem(KernelT kernel, int grid, int threads, size_t smem, cudaStream_t st,
                             const GemvParams& p) {
    cudaError_t e = ensure_smem_optin(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, dim3(grid), dim3(threads), smem, st, p);
}

using GemvKernel = void (*)(const GemvParams);
using GroupKernel = void (*)(const GroupParams);

template <int LPR, int XM, int WB>
GemvKernel small_kernel_for(int mt, int r) {
    if (mt == 1 && r == 1) return gemv_small_kernel<LPR, 1, 1, XM, WB>;
    if (mt == 1 && r == 2) return gemv_small_kernel<LPR, 1, 2, XM, WB>;
    if (mt == 1 && r == 4) return gemv_small_kernel<LPR, 1, 4, XM, WB>;
    if (mt == 2 && r == 1) return gemv_small_kernel<LPR, 2, 1, XM, WB>;
    if (mt == 2 && r == 2) return gemv_small_kernel<LPR, 2, 2, XM, WB>;
    return gemv_small_kernel<LPR, 4, 1, XM, WB>;
}

template <int XM, int WB>
GemvKernel small_kernel_for(int lpr, int mt, int r) {
    if (lpr == 32) return small_kernel_for<32, XM, WB>(mt, r);
    if (lpr == 16) return small_kernel_for<16, XM, WB>(mt, r);
    return small_kernel_for<8, XM, WB>(mt, r);
}

template <int WB>
GemvKernel small_kernel_for_mode(int x_mode, int lpr, int mt, int r) {
    return x_mode == X_QUANTISED ? small_kernel_for<X_QUANTISED, WB>(lpr, mt, r)
           : x_mode == X_F32     ? small_kernel_for<X_F32, WB>(lpr, mt, r)
                                 : small_kernel_for<X_BF16, WB>(lpr, mt, r);
}

// Ring geometry for a CTA slab of `rows_per_cta` rows and `ring_bytes` of
// space: chunks of a power-of-two number of rows (about 8 KiB), one slot per
// chunk when the slab fits, otherwise a ring of as many slots as fit.
void ring_geometry(GemvParams& p, int rows_per_cta, int ring_bytes) {
    const int RB = p.rb;
    const int cap = std::max(1, std::min(rows_per_cta, GEMV_CHUNK_TARGET / RB));
    p.rpc_shift = 0;
    while ((2 << p.rpc_shift) <= cap) ++p.rpc_shift;
    p.rpc = 1 << p.rpc_shift;
    p.stage_stride = p.rpc * RB;  // multiple of 16 (K % 64 == 0); >= one row (<= 64 KiB)
    const int nchunks = (rows_per_cta + p.rpc - 1) / p.rpc;
    const int fit = std::max(1, std::min(ring_bytes / p.stage_stride, GEMV_MAX_STAGES));
    p.reuse = nchunks > fit;
    p.stages = p.reuse ? fit : nchunks;
}

int small_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : 4; }

struct SmallShape {
    int lpr, r, cwarps, grid;
    size_t smem;
};

// Launch shape and ring geometry of the small kernel for problem p when
// `co_resident` CTAs share an SM (sets the ring fields of p).
SmallShape configure_small(GemvParams& p, const DevInfo& dev, int co_resident) {
    const int K = p.K, N = p.N;
    const int grid = std::max(1, std::min(N, dev.num_sms));
    const int rows_per_cta = (N + grid - 1) / grid;
    const int K4 = p.rb / 16;  // 16-byte groups of packed weights per row
    const int mt = small_mt(p.M);
    // Launch shape (measured on B200 over lanes-per-row x rows-per-team x
    // K-slices x warps for the 4096x11008 and 11008x4096 decode shapes):
    // about ten consumer warps, two rows per team (one when M > 2), and the
    // widest team for which every row of the CTA still fits one pass.
    const int cw_target = 10;
    int r = std::max(1, 2 / mt);
    const int teams_needed = (rows_per_cta + r - 1) / r;
    int lpr = 8;
    for (int l : {32, 16, 8}) {
        if (teams_needed * l <= cw_target * 32) {
            lpr = l;
            break;
        }
    }
    int ks = 1;
    if (rows_per_cta <= GEMV_KS_MAX_ROWS && lpr == 32 && (cw_target * 32 / lpr) * r >= 2 * rows_per_cta)
        ks = 2;  // few rows: split K so every warp has work
    p.ks = ks;
    p.slice4 = (K4 + ks - 1) / ks;
    const int items = (rows_per_cta + r - 1) / r * ks;
    int cwarps = std::max(1, std::min(cw_target, (items * lpr + 31) / 32));
    p.xq_bytes = (mt * K + 127) / 128 * 128;
    // leave room for the other CTAs on the same SM
    const int budget = (dev.max_smem_optin - 1024) / co_resident;
    const int ring_bytes = std::max(budget - GEMV_HDR - p.xq_bytes, 2 * p.rb);
    ring_geometry(p, rows_per_cta, ring_bytes);
    if (p.reuse) {
        // one team per warp, and the rows of one iteration (ceil(teams / ks) * r)
        // within (stages - 1) * rpc so that they never wrap onto a slot twice
        const int window = std::max(1, (p.stages - 1) * p.rpc);
        lpr = 32;
        r = std::min(r, window);
        while (r > 1 && (r & (r - 1))) --r;  // keep r in {1, 2, 4}
        const int teams_max = std::max(1, window / r * ks);
        cwarps = std::max(1, std::min(cwarps, teams_max));
        // teams per iteration a multiple (or divisor) of ks: iterations then
        // start on row-group boundaries
        if (cwarps >= ks)
            cwarps = cwarps / ks * ks;
        else
            while (ks % cwarps) --cwarps;
    }
    SmallShape sh;
    sh.lpr = lpr;
    sh.r = r;
    sh.cwarps = cwarps;
    sh.grid = grid;
    sh.smem = GEMV_HDR + p.xq_bytes + (size_t)p.stages * p.stage_stride;
    return sh;
}

bool small_ok(int M, int K) { return M <= GEMV_SMALL_MAX_M && small_mt(M) * K <= GEMV_XQ_SMEM_MAX; }

cudaError_t launch_gemv_impl(GemvParams& p, const DevInfo& dev, cudaStream_t st) {
    const int M = p.M, N = p.N;
    if (small_ok(M, p.K)) {
        const SmallShape sh = configure_small(p, dev, GEMV_CO_RESIDENT);
        if (take_wait_expiry_request()) {  // test hook: the first CTA never receives its weights
            p.wait_limit = 100000;
            p.stall_cta = 0;
        }
        const int mt = small_mt(M);
        GemvKernel k = small_kernel_for_mode<2>(p.x_mode, sh.lpr, mt, sh.r);
        return launch_with_smem(k, sh.grid, (sh.cwarps + 1) * 32, sh.smem, st, p);
    }
    if (p.x_mode != X_QUANTISED) return cudaErrorInvalidValue;  // callers quantise first
    const int grid = std::max(1, std::min(N, dev.num_sms));
    const int rows_per_cta = (N + grid - 1) / grid;
    p.xq_bytes = 0;
    ring_geometry(p, rows_per_cta, dev.max_smem_optin - GEMV_HDR);
    p.wave = p.reuse ? std::max(1, std::min(GEMV_MT_CWARPS, (p.stages - 1) * p.rpc)) : GEMV_MT_CWARPS;
    const size_t smem = GEMV_HDR + (size_t)p.stages * p.stage_stride;
    const int threads = (GEMV_MT_CWARPS + 1) * 32;
    if (M <= 1) return launch_with_smem(gemv_mt_kernel<1>, grid, threads, smem, st, p);
    if (M <= 2) return launch_with_smem(gemv_mt_kernel<2>, grid, threads, smem, st, p);
    if (M <= 4) return launch_with_smem(gemv_mt_kernel<4>, grid, threads, smem, st, p);
    return launch_with_smem(gemv_mt_kernel<8>, grid, threads, smem, st, p);
}

template <int XM>
GroupKernel group_kernel_for(int mt) {
    if (mt == 1) return gemv_group_kernel<1, 2, XM>;
    if (mt == 2) return gemv_group_kernel<2, 1, XM>;
    return gemv_group_kernel<4, 1, XM>;
}

GemvParams make_params(const int8_t* x_q, const float* gamma, int M, int K, const uint32_t* W_p, const float* beta,
                       int N, void* y, YMode mode) {
    GemvParams p = {};
    p.wait_limit = WAIT_LIMIT_CYCLES;
    p.stall_cta = -1;
    p.x_q = x_q;
    p.gamma = gamma;
    p.W_p = W_p;
    p.beta = beta;
    p.y = y;
    p.M = M;
    p.K = K;
    p.N = N;
    p.mode = mode;
    p.x_mode = X_QUANTISED;
    p.rb = K / 4;
    return p;
}

}  // namespace

cudaError_t launch_gemv(const int8_t* x_q, const float* gamma, int M, int K, const uint32_t* W_p, const float* beta,
                        int N, void* y, YMode mode, const DevInfo& dev, cudaStream_t st) {
    GemvParams p = make_params(x_q, gamma, M, K, W_p, beta, N, y, mode);
    return launch_gemv_impl(p, dev, st);
}

bool gemv_fused_quant_ok(long long M, long long K) {
    return M <= GEMV_SMALL_MAX_M && small_mt((int)M) * K <= GEMV_XQ_SMEM_MAX;
}

int gemv_group_max() { return GEMV_GROUP_MAX; }

cudaError_t launch_gemv_fused_group(const GemvProblem* probs, int count, int M, int x_dtype, YMode mode,
                                    const DevInfo& dev, cudaStream_t st) {
    // x_dtype: 0 fp32, 1 bf16 (quantiser fused), 2 int8 x_q with gamma
    const int xm = x_dtype == 2 ? X_QUANTISED : x_dtype == 1 ? X_BF16 : X_F32;
    if (count < 1 || count > GEMV_GROUP_MAX) return cudaErrorInvalidValue;
    GroupParams g = {};
    g.count = count;
    int threads = 32;
    size_t smem = 0;
    int cta = 0;
    for (int i = 0; i < count; ++i) {
        const GemvProblem& q = probs[i];
        if (!small_ok(M, q.K)) return cudaErrorInvalidValue;
        GemvParams p = make_params(nullptr, nullptr, M, q.K, q.W_p, q.beta, q.N, q.y, mode);
        if (xm == X_QUANTISED) {
            p.x_q = static_cast<const int8_t*>(q.x);
            p.gamma = q.gamma;
        } else {
            p.x = q.x;
        }
        p.x_mode = xm;
        // the problems of the group share each SM (one CTA each)
        const SmallShape sh = configure_small(p, dev, count);
        g.prob[i] = p;
        g.lpr[i] = sh.lpr;
        g.cta0[i] = cta;
        cta += sh.grid;
        threads = std::max(threads, (sh.cwarps + 1) * 32);
        smem = std::max(smem, sh.smem);
    }
    g.cta0[count] = cta;
    if (take_wait_expiry_request()) {  // test hook: the first CTA never receives its weights
        g.prob[0].wait_limit = 100000;
        g.prob[0].stall_cta = 0;
    }
    const int mt = small_mt(M);
    GroupKernel k = xm == X_QUANTISED ? group_kernel_for<X_QUANTISED>(mt)
                    : xm == X_BF16    ? group_kernel_for<X_BF16>(mt)
                                      : group_kernel_for<X_F32>(mt);
    cudaError_t e = ensure_smem_optin(reinterpret_cast<const void*>(k), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(cta), dim3(threads), smem, st, g);
}

bool gemv_bits_ok(long long M, long long K) { return gemv_fused_quant_ok(M, K); }

cudaError_t launch_gemv_bits(const void* x, int x_dtype, const float* gamma, int M, int K, const uint32_t* W_p,
                             const float* beta, int N, void* y, YMode mode, const DevInfo& dev, cudaStream_t st) {
    // x_dtype: 0 fp32, 1 bf16 (quantiser fused), 2 int8 x_q with gamma
    if (!small_ok(M, K)) return cudaErrorInvalidValue;
    GemvParams p = make_params(nullptr, nullptr, M, K, W_p, beta, N, y, mode);
    p.rb = K / 8;
    if (x_dtype == 2) {
        p.x_q = static_cast<const int8_t*>(x);
        p.gamma = gamma;
    } else {
        p.x = x;
        p.x_mode = x_dtype == 1 ? X_BF16 : X_F32;
    }
    const SmallShape sh = configure_small(p, dev, GEMV_CO_RESIDENT);
    GemvKernel k = small_kernel_for_mode<1>(p.x_mode, sh.lpr, small_mt(M), sh.r);
    return launch_with_smem(k, sh.grid, (sh.cwarps + 1) * 32, sh.smem, st, p);
}

cudaError_t launch_gemv_fused(const void* x, bool bf16, int M, int K, const uint32_t* W_p, const float* beta, int N,
                              void* y, YMode mode, const DevInfo& dev, cudaStream_t st) {
    GemvParams p = make_params(nullptr, nullptr, M, K, W_p, beta, N, y, mode);
    p.x = x;
    p.x_mode = bf16 ? X_BF16 : X_F32;
    return launch_gemv_impl(p, dev, st);
}

}  // namespace bl
