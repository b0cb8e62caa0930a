// k_gemv1.cu -- decode BitLinear forward for ONE token, up to eight
// independent projections in one launch, on CUDA cores.
//
// DataCamp blog "MatMul-free language models", section "MatMul vervangen
// door ternaire bewerkingen": with weights in {-1, 0, +1} the layer is a
// ternary accumulation.  unite.ai page, "Mathematische Grundlagen", eq. 2
// (per-token absmax int8 quantiser) and eq. 3 "BitLinear-Betrieb" (rescale by
// beta * gamma / Q_b).
//
// A single token's projection moves its packed weights once and does almost
// nothing else, so a decode step is a stream of HBM bytes with a short,
// latency-bound prologue (the activation quantiser) that can only start once
// the preceding kernel has finished.  The design hides everything but that
// prologue behind the weight stream of the NEXT launch:
//
//   * one CTA per SM owns a contiguous slab of rows of every problem;
//   * a CTA takes at most half of an SM (512 threads, 64 registers, about
//     113 KB of shared memory), so the following launch's CTA is resident
//     beside it as soon as this one has started (programmatic dependent
//     launch) and fills its own weight rings while this one computes;
//   * each problem has its own ring of chunk slots (a power-of-two number of
//     rows, about 8 KB), fed by 1-D bulk copies from one producer thread that
//     never waits for the preceding kernel (weights and beta are inputs that
//     no in-flight kernel writes);
//   * a consumer warp is bound to one K slice (<= 64 groups of 16 packed
//     bytes = 4096 trits) of one problem and keeps that slice of x_hat in
//     registers (two 64-byte groups per lane), so the row loop reads only the
//     weights from shared memory: one 16-byte load, four LOP3 and four
//     dp4a.u32.s32 per 64 trits and lane per group;
//   * R rows at a time are finished by one batched shuffle reduction; rows
//     cut into several K slices add their slice sums in shared memory
//     (integer, so the order does not matter) and are written at the end.
//
// The quantiser is the one of the other decode kernels: absmax per token
// over the row (exact, order-free), s = 127 / gamma, codes rint(x s) clamped
// to [-127, 127], row sum of the codes for the c = w + 1 correction.
#include "act_inl.cuh"
#include "common.cuh"
#include "gemv_inl.cuh"
#include "kernels.cuh"

namespace bl {

namespace {

constexpr int G1_MAX_PROBS = 8;
constexpr int G1_CWARPS = 15;                     // consumer warps (warp 0 produces)
constexpr int G1_THREADS = (G1_CWARPS + 1) * 32;  // 512: two CTAs fit an SM by registers
constexpr int G1_MAX_BARS = 64;                   // ring slots over all problems
constexpr int G1_PART_MAX = 512;                  // slice sums of K-sliced rows per CTA
constexpr int G1_SLICE_UNITS = 64;                // 16-byte packed groups per K slice (2 per lane)
constexpr int G1_CHUNK_TARGET = 8192;             // bytes per ring slot (about)
constexpr int G1_XC = 2;                          // activation chunks cached per staging thread
constexpr int G1_MAX_SUMK = G1_XC * G1_CWARPS * 32 * 16;  // every chunk cached: sum of K <= 15360

struct G1Prob {
    const void* x;       // fp32 / bf16 activations, or int8 x_q (with gamma)
    const float* gamma;  // x_q mode only
    const uint32_t* W_p;
    const float* beta;
    void* y;
    int K, N;
    int rb;         // bytes per packed row (K / 4)
    int rpc_shift;  // log2(rows per ring slot)
    int slot;       // bytes per ring slot
    int stages;     // ring slots
    int ring_off;   // shared-memory offset of the ring
    int bar0;       // first barrier of the ring
    int xq_off;     // shared-memory offset of x_hat (K bytes)
    int nslice;     // K slices; rows with more than one add slice sums in part[]
    int slice_w;    // 16-byte groups per slice (the last slice may be shorter)
    int part_off;   // first part[] entry of this problem's rows
};

struct G1Params {
    G1Prob prob[G1_MAX_PROBS];
    int count;
    int x_mode;  // X_QUANTISED, X_F32 or X_BF16
    int mode;    // Y_F32, Y_BF16 or Y_ACC
    int sliced;  // any problem with nslice > 1
    long long wait_limit;  // SM cycles before a wait gives up
    int stall_cta;         // test hook: this CTA's producer issues nothing (-1: none)
    // role of consumer warp w: problem, K slice, index in the (problem, slice)
    // group, group size, rows per batch (1, 2 or 4)
    unsigned char wp[G1_CWARPS], ws[G1_CWARPS], wj[G1_CWARPS], wn[G1_CWARPS], wr[G1_CWARPS];
};

struct G1Shared {
    uint64_t full[G1_MAX_BARS];
    uint64_t empty[G1_MAX_BARS];
    int abort_flag;
    int rowsum[G1_MAX_PROBS];
    float beta[G1_MAX_PROBS];
    float fscale[G1_MAX_PROBS];
    unsigned red[G1_CWARPS][G1_MAX_PROBS];
    int part[G1_PART_MAX];
};
constexpr int G1_HDR = (int)((sizeof(G1Shared) + 127) / 128 * 128);

__device__ __forceinline__ void g1_rows(const G1Prob& q, int cta, int ncta, int& r0, int& n) {
    const long long N = q.N;
    r0 = (int)((N * cta) / ncta);
    n = (int)((N * (cta + 1)) / ncta) - r0;
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Issue chunk k of problem q (rows [k << rpc_shift, ...) of this CTA's slab).
__device__ __forceinline__ void g1_issue(const G1Prob& q, G1Shared& sh, unsigned char* smem, int r0, int n, int k,
                                         uint64_t pol) {
    const int st = k % q.stages;
    const int rows = min(1 << q.rpc_shift, n - (k << q.rpc_shift));
    const uint32_t bytes = (uint32_t)rows * q.rb;
    uint64_t* full = &sh.full[q.bar0 + st];
    mbar_arrive_expect_tx(full, bytes);
    const unsigned char* src =
        reinterpret_cast<const unsigned char*>(q.W_p) + ((long long)r0 + ((long long)k << q.rpc_shift)) * q.rb;
    bulk_g2s(smem + q.ring_off + (size_t)st * q.slot, src, bytes, full, pol);
}

// Producer thread: every chunk of every problem, problems interleaved, a
// slot reused once all its (row, slice) consumers have arrived.  Polls the
// rings so that one problem's full ring never holds up another's.
__device__ void g1_produce(const G1Params& g, G1Shared& sh, unsigned char* smem, int cta, int ncta, int first_k) {
    const uint64_t pol = policy_evict_first();
    int next[G1_MAX_PROBS], nch[G1_MAX_PROBS], r0[G1_MAX_PROBS], nr[G1_MAX_PROBS];
    int left = 0;
#pragma unroll
    for (int i = 0; i < G1_MAX_PROBS; ++i) {
        next[i] = nch[i] = r0[i] = nr[i] = 0;
        if (i < g.count) {
            g1_rows(g.prob[i], cta, ncta, r0[i], nr[i]);
            nch[i] = (nr[i] + (1 << g.prob[i].rpc_shift) - 1) >> g.prob[i].rpc_shift;
            next[i] = min(first_k, nch[i]);
            left += nch[i] - next[i];
        }
    }
    long long t0 = -1;
    while (left > 0) {
        bool progress = false;
#pragma unroll
        for (int i = 0; i < G1_MAX_PROBS; ++i) {
            if (i >= g.count) break;
            const G1Prob& q = g.prob[i];
            const int k = next[i];
            if (k >= nch[i]) continue;
            if (k >= q.stages && !mbar_test(&sh.empty[q.bar0 + k % q.stages], ((k / q.stages) - 1) & 1)) continue;
            g1_issue(q, sh, smem, r0[i], nr[i], k, pol);
            next[i] = k + 1;
            --left;
            progress = true;
        }
        if (progress) {
            t0 = -1;
        } else {
            if (*(volatile int*)&sh.abort_flag) return;
            const long long t = clock64();
            if (t0 < 0) t0 = t;
            if (t - t0 > g.wait_limit) {
                set_dev_error(DEV_ERR_TIMEOUT);
                sh.abort_flag = 1;
                return;
            }
        }
    }
}

// Wait for the phase of the given parity, at most `limit` SM cycles; false
// (and the device error word raised) if it did not complete in time.
__device__ __forceinline__ bool g1_wait(uint64_t* bar, uint32_t parity, long long limit) {
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

__device__ __forceinline__ void g1_consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(G1_CWARPS * 32) : "memory");
}

__device__ __forceinline__ void g1_store(const G1Params& g, const G1Prob& q, int n, int acc, float f) {
    if (g.mode == Y_ACC) {
        reinterpret_cast<int*>(q.y)[n] = acc;
    } else {
        const float v = __fmul_rn((float)acc, f);
        if (g.mode == Y_F32)
            reinterpret_cast<float*>(q.y)[n] = v;
        else
            reinterpret_cast<uint16_t*>(q.y)[n] = f32_to_bf16_rn(v);
    }
}

// Consumers: quantise the token of every problem into shared memory (codes
// in k order, row sums, rescale factors).  Every 16-element chunk of the
// concatenated activations is loaded once into registers and serves both the
// absmax pass and the code pass.
template <int XM>
__device__ __forceinline__ void g1_stage(const G1Params& g, G1Shared& sh, unsigned char* smem, int ctid) {
    constexpr int CT = G1_CWARPS * 32;
    const int lane = ctid & 31, warp = ctid >> 5;
    XChunk<XM> cache[G1_XC];
    int cp[G1_XC], cg[G1_XC];
#pragma unroll
    for (int i = 0; i < G1_XC; ++i) {
        int gi = ctid + i * CT;
        int p = -1;
        for (int j = 0; j < g.count; ++j) {
            const int gj = g.prob[j].K >> 4;
            if (p < 0 && gi < gj) p = j;
            if (p < 0) gi -= gj;
        }
        cp[i] = p;
        cg[i] = gi;
        if (p >= 0) ld_chunk<XM>(g.prob[p].x, gi, cache[i]);
    }
    float s[G1_XC];
#pragma unroll
    for (int i = 0; i < G1_XC; ++i) s[i] = 0.0f;
    if constexpr (XM != X_QUANTISED) {
        unsigned am[G1_XC];
#pragma unroll
        for (int i = 0; i < G1_XC; ++i) am[i] = cp[i] >= 0 ? chunk_absmax<XM>(cache[i], 0u) : 0u;
        for (int p = 0; p < g.count; ++p) {
            unsigned a = 0u;
#pragma unroll
            for (int i = 0; i < G1_XC; ++i)
                if (cp[i] == p) a = max(a, am[i]);
            a = __reduce_max_sync(0xffffffffu, a);
            if (lane == 0) sh.red[warp][p] = a;
        }
        g1_consumer_sync();
#pragma unroll
        for (int i = 0; i < G1_XC; ++i) {
            if (cp[i] >= 0) {
                unsigned a = 0u;
                for (int w = 0; w < G1_CWARPS; ++w) a = max(a, sh.red[w][cp[i]]);
                s[i] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(a), 1e-5f));
            }
        }
        if (ctid < g.count) {
            unsigned a = 0u;
            for (int w = 0; w < G1_CWARPS; ++w) a = max(a, sh.red[w][ctid]);
            const float gam = fmaxf(__uint_as_float(a), 1e-5f);
            sh.fscale[ctid] = g.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(sh.beta[ctid], gam), 127.0f);
        }
    } else if (ctid < g.count) {
        sh.fscale[ctid] =
            g.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(sh.beta[ctid], __ldg(g.prob[ctid].gamma)), 127.0f);
    }
    for (int i = ctid; i < G1_PART_MAX; i += CT) sh.part[i] = 0;
    int rs[G1_XC];
#pragma unroll
    for (int i = 0; i < G1_XC; ++i) {
        rs[i] = 0;
        if (cp[i] >= 0) {
            const int4 q = chunk_codes<XM>(cache[i], s[i]);
            rs[i] = bytesum_s8(q.x) + bytesum_s8(q.y) + bytesum_s8(q.z) + bytesum_s8(q.w);
            *reinterpret_cast<int4*>(smem + g.prob[cp[i]].xq_off + 16 * cg[i]) = q;
        }
    }
    for (int p = 0; p < g.count; ++p) {
        int v = 0;
#pragma unroll
        for (int i = 0; i < G1_XC; ++i)
            if (cp[i] == p) v += rs[i];
        v = __reduce_add_sync(0xffffffffu, v);
        if (lane == 0 && v != 0) atomicAdd(&sh.rowsum[p], v);
    }
    g1_consumer_sync();
}

// One consumer warp's share: rows b*R .. b*R+R-1 for batches b = j, j + n, ...
// of problem q, K slice sl.  UPL = 16-byte groups per lane (1 or 2).
template <int R, int UPL>
__device__ __forceinline__ void g1_rows_loop(const G1Params& g, const G1Prob& q, G1Shared& sh, unsigned char* smem,
                                             int pi, int sl, int j, int n, int r0, int nrows) {
    const int lane = threadIdx.x & 31;
    const int U = q.K >> 6;
    const int u0 = sl * q.slice_w;
    const int width = min(q.slice_w, U - u0);
    const bool ha = lane < width;
    const bool hb = UPL == 2 && lane + 32 < width;
    // x_hat of this lane's groups: 64 codes each, k = 64u .. 64u + 63
    int4 xa[4], xb[4];
    const int4* xq = reinterpret_cast<const int4*>(smem + q.xq_off);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xa[i] = ha ? xq[4 * (u0 + lane) + i] : make_int4(0, 0, 0, 0);
        xb[i] = hb ? xq[4 * (u0 + lane + 32) + i] : make_int4(0, 0, 0, 0);
    }
    const int rmask = (1 << q.rpc_shift) - 1;
    const float f = sh.fscale[pi];
    const int rowsum = sh.rowsum[pi];
    for (int b = j; b * R < nrows; b += n) {
        const int i0 = b * R;
        const int nv = min(R, nrows - i0);
        bool ok = !*(volatile int*)&sh.abort_flag;
        int vals[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            vals[r] = 0;
            if (r < nv && ok) {
                const int i = i0 + r;
                const int k = i >> q.rpc_shift;
                const int st = k % q.stages;
                if (!g1_wait(&sh.full[q.bar0 + st], (uint32_t)((k / q.stages) & 1), g.wait_limit)) {
                    sh.abort_flag = 1;
                    ok = false;
                } else {
                    const uint4* wr = reinterpret_cast<const uint4*>(smem + q.ring_off + (size_t)st * q.slot +
                                                                     (size_t)(i & rmask) * q.rb) +
                                      u0;
                    const uint4 wa = ha ? wr[lane] : make_uint4(0u, 0u, 0u, 0u);
                    const uint4 wb = hb ? wr[lane + 32] : make_uint4(0u, 0u, 0u, 0u);
                    int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
                    word_dot(wa.x, xa[0].x, xa[0].y, xa[0].z, xa[0].w, a0, a1, a2, a3);
                    word_dot(wa.y, xa[1].x, xa[1].y, xa[1].z, xa[1].w, a0, a1, a2, a3);
                    word_dot(wa.z, xa[2].x, xa[2].y, xa[2].z, xa[2].w, a0, a1, a2, a3);
                    word_dot(wa.w, xa[3].x, xa[3].y, xa[3].z, xa[3].w, a0, a1, a2, a3);
                    if (UPL == 2) {
                        word_dot(wb.x, xb[0].x, xb[0].y, xb[0].z, xb[0].w, a0, a1, a2, a3);
                        word_dot(wb.y, xb[1].x, xb[1].y, xb[1].z, xb[1].w, a0, a1, a2, a3);
                        word_dot(wb.z, xb[2].x, xb[2].y, xb[2].z, xb[2].w, a0, a1, a2, a3);
                        word_dot(wb.w, xb[3].x, xb[3].y, xb[3].z, xb[3].w, a0, a1, a2, a3);
                    }
                    vals[r] = combine4(a0, a1, a2, a3);
                }
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        int which;
        const int tot = team_reduce<32, R>(vals, lane, which);
        if (ok && lane == which * (32 / R) && which < nv) {
            const int i = i0 + which;
            if (q.nslice == 1)
                g1_store(g, q, r0 + i, tot - rowsum, f);
            else
                atomicAdd(&sh.part[q.part_off + i], tot);
            mbar_arrive(&sh.empty[q.bar0 + (i >> q.rpc_shift) % q.stages]);
        }
    }
}

template <int XM>
__global__ void __launch_bounds__(G1_THREADS, 2) gemv1_kernel(const __grid_constant__ G1Params g) {
    extern __shared__ __align__(128) unsigned char smem[];
    G1Shared& sh = *reinterpret_cast<G1Shared*>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x, ncta = gridDim.x;
    if (threadIdx.x == 0) {
        for (int p = 0; p < g.count; ++p) {
            const G1Prob& q = g.prob[p];
            for (int s = 0; s < q.stages; ++s) {
                mbar_init(&sh.full[q.bar0 + s], 1);
                mbar_init(&sh.empty[q.bar0 + s], (1u << q.rpc_shift) * q.nslice);
            }
            sh.rowsum[p] = 0;
            // beta and W_p are weight inputs, not written by the preceding
            // kernel: read before waiting for it
            sh.beta[p] = g.mode == Y_ACC ? 0.0f : __ldg(q.beta);
        }
        sh.abort_flag = 0;
        fence_mbar_init();
        // the first chunk of every problem is in flight before the CTA barrier
        const uint64_t pol = policy_evict_first();
        for (int p = 0; p < g.count && cta != g.stall_cta; ++p) {
            int r0, n;
            g1_rows(g.prob[p], cta, ncta, r0, n);
            if (n > 0) g1_issue(g.prob[p], sh, smem, r0, n, 0, pol);
        }
    }
    __syncthreads();
    pdl_launch_dependents();
    if (warp == 0) {
        if (lane == 0 && cta != g.stall_cta) g1_produce(g, sh, smem, cta, ncta, 1);
        return;
    }
    pdl_wait();
    const int cw = warp - 1;
    g1_stage<XM>(g, sh, smem, threadIdx.x - 32);
    const int pi = g.wp[cw];
    if (pi < g.count) {
        const G1Prob& q = g.prob[pi];
        int r0, n;
        g1_rows(q, cta, ncta, r0, n);
        const int sl = g.ws[cw], j = g.wj[cw], nn = g.wn[cw], R = g.wr[cw];
        const bool two = min(q.slice_w, (q.K >> 6) - sl * q.slice_w) > 32;  // groups per lane: 2 or 1
        if (R == 4)
            two ? g1_rows_loop<4, 2>(g, q, sh, smem, pi, sl, j, nn, r0, n)
                : g1_rows_loop<4, 1>(g, q, sh, smem, pi, sl, j, nn, r0, n);
        else if (R == 2)
            two ? g1_rows_loop<2, 2>(g, q, sh, smem, pi, sl, j, nn, r0, n)
                : g1_rows_loop<2, 1>(g, q, sh, smem, pi, sl, j, nn, r0, n);
        else
            two ? g1_rows_loop<1, 2>(g, q, sh, smem, pi, sl, j, nn, r0, n)
                : g1_rows_loop<1, 1>(g, q, sh, smem, pi, sl, j, nn, r0, n);
    }
    if (g.sliced) {  // every slice of every row is in: finish the sliced rows
        g1_consumer_sync();
        if (*(volatile int*)&sh.abort_flag) return;
        const int ctid = threadIdx.x - 32;
        for (int p = 0; p < g.count; ++p) {
            const G1Prob& q = g.prob[p];
            if (q.nslice == 1) continue;
            int r0, n;
            g1_rows(q, cta, ncta, r0, n);
            const float f = sh.fscale[p];
            const int rowsum = sh.rowsum[p];
            for (int i = ctid; i < n; i += G1_CWARPS * 32) g1_store(g, q, r0 + i, sh.part[q.part_off + i] - rowsum, f);
        }
    }
}

// ------------------------------------------------------------------- host

// Estimated issue slots of one warp of a (problem, slice) group of n warps
// working on `rows` rows with `upl` groups per lane, and the batch size that
// minimises it.
int g1_cost(int rows, int upl, int n, int& best_r) {
    int best = 1 << 30;
    best_r = 1;
    for (int R : {4, 2, 1}) {
        const int batches = (rows + R - 1) / R;
        const int per_warp = (batches + n - 1) / n * R;
        const int red = R == 1 ? 10 : R == 2 ? 5 : 3;  // shuffle-reduction steps per row
        const int c = per_warp * (upl * 33 + 4 + red);
        if (c < best) {
            best = c;
            best_r = R;
        }
    }
    return best;
}

}  // namespace

// Plan the launch; false when the problem set does not suit the kernel (the
// caller then uses the general small-M kernel).
static bool g1_plan(const GemvProblem* probs, int count, int x_mode, YMode mode, const DevInfo& dev, G1Params& g,
                    int& grid, size_t& smem) {
    if (count < 1 || count > G1_MAX_PROBS) return false;
    g = {};
    g.count = count;
    g.x_mode = x_mode;
    g.mode = mode;
    int sumK = 0, maxN = 0, pairs = 0;
    for (int i = 0; i < count; ++i) {
        const int K = probs[i].K;
        if (K % 64 || K < 64 * 32) return false;  // a slice narrower than a warp idles lanes
        sumK += K;
        maxN = std::max(maxN, probs[i].N);
        pairs += (K / 64 + G1_SLICE_UNITS - 1) / G1_SLICE_UNITS;
    }
    if (sumK > G1_MAX_SUMK || pairs > G1_CWARPS) return false;
    grid = std::max(1, std::min(dev.num_sms, maxN));
    // two CTAs per SM: the shared memory of one SM (228 KB) halved, less the
    // 1 KB the hardware reserves per CTA
    const int budget = std::min(dev.max_smem_optin, 233472 / 2 - 1024);
    int off = G1_HDR;
    long long slab_bytes[G1_MAX_PROBS];
    long long total = 0;
    int part = 0;
    for (int i = 0; i < count; ++i) {
        G1Prob& q = g.prob[i];
        const GemvProblem& s = probs[i];
        q.x = s.x;
        q.gamma = s.gamma;
        q.W_p = s.W_p;
        q.beta = s.beta;
        q.y = s.y;
        q.K = s.K;
        q.N = s.N;
        q.rb = s.K / 4;
        q.xq_off = off;
        off += (s.K + 127) / 128 * 128;
        const int U = s.K / 64;
        q.nslice = (U + G1_SLICE_UNITS - 1) / G1_SLICE_UNITS;
        q.slice_w = (U + q.nslice - 1) / q.nslice;
        const int rows_max = (s.N + grid - 1) / grid;
        int rpc = 1;
        while (rpc * 2 * q.rb <= G1_CHUNK_TARGET && rpc * 2 <= std::max(1, rows_max)) rpc *= 2;
        q.rpc_shift = 0;
        while ((1 << q.rpc_shift) < rpc) ++q.rpc_shift;
        q.slot = rpc * q.rb;
        if (q.nslice > 1) {
            q.part_off = part;
            part += rows_max;
        }
        slab_bytes[i] = (long long)rows_max * q.rb;
        total += slab_bytes[i];
        g.sliced |= q.nslice > 1;
    }
    if (part > G1_PART_MAX) return false;
    const int ring_budget = budget - off;
    if (ring_budget <= 0) return false;
    int bars = 0;
    for (int i = 0; i < count; ++i) {
        G1Prob& q = g.prob[i];
        const int rows_max = (q.N + grid - 1) / grid;
        const int nch = (rows_max + (1 << q.rpc_shift) - 1) >> q.rpc_shift;
        const long long share = (long long)ring_budget * slab_bytes[i] / std::max(1LL, total);
        int st = (int)std::min<long long>(share / q.slot, nch);
        // a batch of up to 4 rows spans at most 4 / rpc + 1 chunks; the ring
        // must hold that many so that a warp never waits on a chunk whose
        // slot it still holds
        const int span = std::min(nch, 4 / (1 << q.rpc_shift) + 1 + ((4 % (1 << q.rpc_shift)) ? 1 : 0));
        if (st < span) return false;
        q.stages = st;
        q.ring_off = off;
        off += st * q.slot;
        q.bar0 = bars;
        bars += st;
    }
    if (bars > G1_MAX_BARS || off > budget) return false;
    // consumer warps: one per (problem, slice) to start with, the rest to the
    // group whose slowest warp has the most work
    struct Pair {
        int p, s, rows, upl, n, r;
    };
    Pair pr[G1_CWARPS];
    int np = 0;
    for (int i = 0; i < count; ++i) {
        const G1Prob& q = g.prob[i];
        const int U = q.K / 64;
        for (int s = 0; s < q.nslice; ++s) {
            const int width = std::min(q.slice_w, U - s * q.slice_w);
            pr[np++] = {i, s, (q.N + grid - 1) / grid, width > 32 ? 2 : 1, 1, 1};
        }
    }
    for (int w = np; w < G1_CWARPS; ++w) {
        int worst = 0, wc = -1;
        for (int k = 0; k < np; ++k) {
            int r;
            const int c = g1_cost(pr[k].rows, pr[k].upl, pr[k].n, r);
            if (c > wc) {
                wc = c;
                worst = k;
            }
        }
        ++pr[worst].n;
    }
    int w = 0;
    for (int k = 0; k < np; ++k) {
        int r;
        g1_cost(pr[k].rows, pr[k].upl, pr[k].n, r);
        for (int j = 0; j < pr[k].n; ++j, ++w) {
            g.wp[w] = (unsigned char)pr[k].p;
            g.ws[w] = (unsigned char)pr[k].s;
            g.wj[w] = (unsigned char)j;
            g.wn[w] = (unsigned char)pr[k].n;
            g.wr[w] = (unsigned char)r;
        }
    }
    smem = (size_t)off;
    return true;
}

bool gemv1_ok(const GemvProblem* probs, int count, int M, const DevInfo& dev) {
    if (M != 1) return false;
    G1Params g;
    int grid;
    size_t smem;
    return g1_plan(probs, count, X_QUANTISED, Y_F32, dev, g, grid, smem);
}

cudaError_t launch_gemv1(const GemvProblem* probs, int count, int x_dtype, YMode mode, const DevInfo& dev,
                         cudaStream_t st) {
    // x_dtype: 0 fp32, 1 bf16 (quantiser fused), 2 int8 x_q with gamma
    const int xm = x_dtype == 2 ? X_QUANTISED : x_dtype == 1 ? X_BF16 : X_F32;
    G1Params g;
    int grid;
    size_t smem;
    if (!g1_plan(probs, count, xm, mode, dev, g, grid, smem)) return cudaErrorInvalidValue;
    g.wait_limit = WAIT_LIMIT_CYCLES;
    g.stall_cta = -1;
    if (take_wait_expiry_request()) {  // test hook: CTA 0 never receives its weights
        g.wait_limit = 100000;
        g.stall_cta = 0;
    }
    auto k = xm == X_QUANTISED ? gemv1_kernel<X_QUANTISED> : xm == X_BF16 ? gemv1_kernel<X_BF16> : gemv1_kernel<X_F32>;
    cudaError_t e = ensure_smem_optin(reinterpret_cast<const void*>(k), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(G1_THREADS), smem, st, g);
}

}  // namespace bl
