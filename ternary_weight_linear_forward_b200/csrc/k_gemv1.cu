// k_gemv1.cu -- decode BitLinear forward for ONE token, up to eight
// independent projections in one launch, on CUDA cores.
//
// DataCamp blog "MatMul-free language models", section "MatMul vervangen
// door ternaire bewerkingen": with weights in {-1, 0, +1} the layer is a
// ternary accumulation.  unite.ai page, "Mathematische Grundlagen", eq. 2
// (per-token absmax int8 quantiser) and eq. 3 "BitLinear-Betrieb" (rescale by
// beta * gamma / Q_b).
//
// A single token's projection moves its packed weights once and does little
// else, so a decode step is a stream of HBM bytes behind a short,
// latency-bound prologue (the activation quantiser) that can only start once
// the preceding kernel has finished.  The design hides everything but that
// prologue behind the weight stream:
//
//   * one CTA per SM owns a contiguous slab of rows of every problem;
//   * a CTA takes at most half of an SM (512 threads, 64 registers, under
//     113 KB of shared memory), so the following launch's CTA is resident
//     beside it as soon as this one has started (programmatic dependent
//     launch) and puts its first weight rows in flight while this one
//     computes;
//   * every warp is bound to one K slice (<= 64 groups of 16 packed bytes =
//     4096 trits) of one problem and keeps that slice of x_hat in registers
//     (one or two 64-byte groups per lane);
//   * every lane streams its own 16-byte groups of the warp's rows with
//     cp.async into a per-warp ring of DEPTH row slots in shared memory, one
//     commit group per row, and reads back only what it copied itself: no
//     barrier and no hand-off between warps, and DEPTH rows of every warp (up
//     to 80 KB per CTA) in flight from the moment the CTA starts.  Copies
//     issued by all 512 threads keep far more requests in flight per SM than
//     one thread's bulk copies, which streamed about 1.3 TB/s here;
//   * per row and lane: one or two 16-byte loads, four LOP3 and four
//     dp4a.u32.s32 per 16 trits; R rows at a time are finished by one batched
//     shuffle reduction; rows cut into several K slices add their slice sums
//     in shared memory (integer, so the order does not matter).
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
constexpr int G1_WARPS = 16;
constexpr int G1_THREADS = G1_WARPS * 32;  // 512: two CTAs fit an SM by registers
constexpr int G1_DEPTH = 5;                // rows in flight per warp
constexpr int G1_SLOT = 1024;              // bytes of a ring slot: one row's slice of <= 64 groups
constexpr int G1_PART_MAX = 512;           // slice sums of K-sliced rows per CTA
constexpr int G1_SLICE_UNITS = 64;         // 16-byte packed groups per K slice (2 per lane)
constexpr int G1_XC = 2;                   // activation chunks cached per staging thread
constexpr int G1_MAX_SUMK = G1_XC * G1_THREADS * 16;  // every chunk cached: sum of K <= 16384

struct G1Prob {
    const void* x;       // fp32 / bf16 activations, or int8 x_q (with gamma)
    const float* gamma;  // x_q mode only
    const uint32_t* W_p;
    const float* beta;
    void* y;
    int K, N;
    int rb;        // bytes per packed row (K / 4)
    int xq_off;    // shared-memory offset of x_hat (K bytes)
    int nslice;    // K slices; rows with more than one add slice sums in part[]
    int slice_w;   // 16-byte groups per slice (the last slice may be shorter)
    int part_off;  // first part[] entry of this problem's rows
};

struct G1Params {
    G1Prob prob[G1_MAX_PROBS];
    int count;
    int x_mode;    // X_QUANTISED, X_F32 or X_BF16
    int mode;      // Y_F32, Y_BF16 or Y_ACC
    int sliced;    // any problem with nslice > 1
    int ring_off;  // shared-memory offset of the per-warp rings
    // role of warp w: problem, K slice, index in the (problem, slice) group,
    // group size, rows per batch (1, 2 or 4)
    unsigned char wp[G1_WARPS], ws[G1_WARPS], wj[G1_WARPS], wn[G1_WARPS], wr[G1_WARPS];
};

struct G1Shared {
    G1Prob prob[G1_MAX_PROBS];  // the problem descriptors, copied from the parameters
    int rowsum[G1_MAX_PROBS];
    float beta[G1_MAX_PROBS];
    float fscale[G1_MAX_PROBS];
    unsigned red[G1_WARPS][G1_MAX_PROBS];
    int part[G1_PART_MAX];
};
constexpr int G1_HDR = (int)((sizeof(G1Shared) + 127) / 128 * 128);

__device__ __forceinline__ void g1_rows(const G1Prob& q, int cta, int ncta, int& r0, int& n) {
    const long long N = q.N;
    r0 = (int)((N * cta) / ncta);
    n = (int)((N * (cta + 1)) / ncta) - r0;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void g1_store(int mode, void* y, int n, int acc, float f) {
    if (mode == Y_ACC) {
        reinterpret_cast<int*>(y)[n] = acc;
    } else {
        const float v = __fmul_rn((float)acc, f);
        if (mode == Y_F32)
            reinterpret_cast<float*>(y)[n] = v;
        else
            reinterpret_cast<uint16_t*>(y)[n] = f32_to_bf16_rn(v);
    }
}

// The rows one warp works on, in order: batches b = j, j + n, ... of R
// consecutive rows; the t-th row of the sequence, or -1 past the slab's end.
struct RowSeq {
    int j, n, R, nrows;
    __device__ __forceinline__ int row(int t) const {
        const int i = (j + (t / R) * n) * R + t % R;
        return i < nrows ? i : -1;
    }
};

// This lane's part of a warp's streaming: its one or two 16-byte groups of
// the warp's K slice in every row.
struct Lane {
    const unsigned char* wslice;  // the slice's first byte in row 0 of the CTA's slab
    unsigned char* ring;          // the warp's ring of DEPTH slots
    int rb, lane;
    bool ha, hb;                  // the lane's first / second group exists

    // put row i in flight into ring slot `slot`; one commit group per call,
    // empty for i < 0
    __device__ __forceinline__ void fetch(int i, int slot) const {
        if (i >= 0) {
            const unsigned char* src = wslice + (size_t)i * rb;
            unsigned char* dst = ring + slot * G1_SLOT;
            if (ha) cp_async16(dst + 16 * lane, src + 16 * lane);
            if (hb) cp_async16(dst + 16 * (lane + 32), src + 16 * (lane + 32));
        }
        cp_async_commit();
    }
};

// Quantise the token of every problem into shared memory (codes in k order,
// row sums, rescale factors).  Every 16-element chunk of the concatenated
// activations is loaded once into registers and serves both the absmax pass
// and the code pass.  Called by all threads (two CTA barriers).
template <int XM>
__device__ __forceinline__ void g1_stage(const G1Params& g, G1Shared& sh, unsigned char* smem) {
    const G1Prob* prob = sh.prob;  // the shared copy: indexed at run time without reloading parameters
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    XChunk<XM> cache[G1_XC];
    int cp[G1_XC], cg[G1_XC];
#pragma unroll
    for (int i = 0; i < G1_XC; ++i) {
        int gi = tid + i * G1_THREADS;
        int p = -1;
        for (int j = 0; j < g.count; ++j) {
            const int gj = prob[j].K >> 4;
            if (p < 0 && gi < gj) p = j;
            if (p < 0) gi -= gj;
        }
        cp[i] = p;
        cg[i] = gi;
        if (p >= 0) ld_chunk<XM>(prob[p].x, gi, cache[i]);
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
        __syncthreads();
#pragma unroll
        for (int i = 0; i < G1_XC; ++i) {
            if (cp[i] >= 0) {
                unsigned a = 0u;
                for (int w = 0; w < G1_WARPS; ++w) a = max(a, sh.red[w][cp[i]]);
                s[i] = __fdiv_rn(127.0f, fmaxf(__uint_as_float(a), 1e-5f));
            }
        }
        if (tid < g.count) {
            unsigned a = 0u;
            for (int w = 0; w < G1_WARPS; ++w) a = max(a, sh.red[w][tid]);
            const float gam = fmaxf(__uint_as_float(a), 1e-5f);
            sh.fscale[tid] = g.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(sh.beta[tid], gam), 127.0f);
        }
    } else if (tid < g.count) {
        sh.fscale[tid] = g.mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(sh.beta[tid], __ldg(prob[tid].gamma)), 127.0f);
    }
    for (int i = tid; i < G1_PART_MAX; i += G1_THREADS) sh.part[i] = 0;
    int rs[G1_XC];
#pragma unroll
    for (int i = 0; i < G1_XC; ++i) {
        rs[i] = 0;
        if (cp[i] >= 0) {
            const int4 q = chunk_codes<XM>(cache[i], s[i]);
            rs[i] = bytesum_s8(q.x) + bytesum_s8(q.y) + bytesum_s8(q.z) + bytesum_s8(q.w);
            *reinterpret_cast<int4*>(smem + prob[cp[i]].xq_off + 16 * cg[i]) = q;
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
    __syncthreads();
}

// One warp's share of problem q, K slice starting at group u0: the rows of
// `seq`, rows 0 .. DEPTH-1 of which are already in flight.  A batch of R
// rows is waited for at once, its words loaded at once and its R dot
// products interleaved (independent chains), then its slots are refilled.
// UPL = 16-byte groups per lane (1 or 2).  No barrier inside.
template <int R, int UPL>
__device__ __forceinline__ void g1_loop(const int mode, const G1Prob& q, const G1Shared& sh,
                                        const unsigned char* smem, int pi, int u0, const RowSeq& seq, int r0,
                                        const Lane& ln) {
    static_assert(R <= G1_DEPTH, "a batch must fit the ring");
    const int lane = ln.lane;
    // loop invariants, read once (q is the shared-memory copy)
    void* const y = q.y;
    const int sliced = q.nslice > 1;
    int* const part = const_cast<int*>(sh.part) + q.part_off;
    int4 xa[4], xb[4];  // x_hat of this lane's groups: 64 codes each, k = 64u .. 64u + 63
    const int4* xq = reinterpret_cast<const int4*>(smem + q.xq_off);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xa[i] = ln.ha ? xq[4 * (u0 + lane) + i] : make_int4(0, 0, 0, 0);
        xb[i] = UPL == 2 && ln.hb ? xq[4 * (u0 + lane + 32) + i] : make_int4(0, 0, 0, 0);
    }
    const float f = sh.fscale[pi];
    const int rowsum = sh.rowsum[pi];
    const int batches = (seq.nrows + R - 1) / R;
    int t = 0;  // rows of the sequence consumed so far
    for (int b = seq.j; b < batches; b += seq.n, t += R) {
        // rows t .. t+R-1 have landed once at most DEPTH - R groups are pending
        cp_async_wait<G1_DEPTH - R>();
        uint4 wa[R], wb[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const unsigned char* w = ln.ring + ((t + r) % G1_DEPTH) * G1_SLOT;
            const bool live = b * R + r < seq.nrows;
            wa[r] = live && ln.ha ? *reinterpret_cast<const uint4*>(w + 16 * lane) : make_uint4(0u, 0u, 0u, 0u);
            wb[r] = UPL == 2 && live && ln.hb ? *reinterpret_cast<const uint4*>(w + 16 * (lane + 32))
                                              : make_uint4(0u, 0u, 0u, 0u);
        }
        int a[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) a[r][0] = a[r][1] = a[r][2] = a[r][3] = 0;
#pragma unroll
        for (int r = 0; r < R; ++r) word_dot(wa[r].x, xa[0].x, xa[0].y, xa[0].z, xa[0].w, a[r][0], a[r][1], a[r][2], a[r][3]);
#pragma unroll
        for (int r = 0; r < R; ++r) word_dot(wa[r].y, xa[1].x, xa[1].y, xa[1].z, xa[1].w, a[r][0], a[r][1], a[r][2], a[r][3]);
#pragma unroll
        for (int r = 0; r < R; ++r) word_dot(wa[r].z, xa[2].x, xa[2].y, xa[2].z, xa[2].w, a[r][0], a[r][1], a[r][2], a[r][3]);
#pragma unroll
        for (int r = 0; r < R; ++r) word_dot(wa[r].w, xa[3].x, xa[3].y, xa[3].z, xa[3].w, a[r][0], a[r][1], a[r][2], a[r][3]);
        if (UPL == 2) {
#pragma unroll
            for (int r = 0; r < R; ++r) word_dot(wb[r].x, xb[0].x, xb[0].y, xb[0].z, xb[0].w, a[r][0], a[r][1], a[r][2], a[r][3]);
#pragma unroll
            for (int r = 0; r < R; ++r) word_dot(wb[r].y, xb[1].x, xb[1].y, xb[1].z, xb[1].w, a[r][0], a[r][1], a[r][2], a[r][3]);
#pragma unroll
            for (int r = 0; r < R; ++r) word_dot(wb[r].z, xb[2].x, xb[2].y, xb[2].z, xb[2].w, a[r][0], a[r][1], a[r][2], a[r][3]);
#pragma unroll
            for (int r = 0; r < R; ++r) word_dot(wb[r].w, xb[3].x, xb[3].y, xb[3].z, xb[3].w, a[r][0], a[r][1], a[r][2], a[r][3]);
        }
        int vals[R];
#pragma unroll
        for (int r = 0; r < R; ++r) vals[r] = combine4(a[r][0], a[r][1], a[r][2], a[r][3]);
        // the batch's words are in registers and used: refill its slots with
        // rows t+DEPTH .. t+DEPTH+R-1
#pragma unroll
        for (int r = 0; r < R; ++r) ln.fetch(seq.row(t + r + G1_DEPTH), (t + r) % G1_DEPTH);
        int which;
        const int tot = team_reduce<32, R>(vals, lane, which);
        const int i = b * R + which;
        if (lane == which * (32 / R) && i < seq.nrows) {
            if (!sliced)
                g1_store(mode, y, r0 + i, tot - rowsum, f);
            else
                atomicAdd(part + i, tot);
        }
    }
    cp_async_wait<0>();  // no copy of this lane is in flight past here
}

template <int XM>
__global__ void __launch_bounds__(G1_THREADS, 2) gemv1_kernel(const __grid_constant__ G1Params g) {
    extern __shared__ __align__(128) unsigned char smem[];
    G1Shared& sh = *reinterpret_cast<G1Shared*>(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x, ncta = gridDim.x;

    const int pi = g.wp[warp];
    int r0, n, u0, width;
    Lane ln;
    {
        const G1Prob& qp = g.prob[pi];  // read once, before the shared copy exists
        g1_rows(qp, cta, ncta, r0, n);
        u0 = g.ws[warp] * qp.slice_w;
        width = min(qp.slice_w, (qp.K >> 6) - u0);  // 16-byte groups of this slice
        ln.wslice = reinterpret_cast<const unsigned char*>(qp.W_p) + (size_t)r0 * qp.rb + 16 * u0;
        ln.rb = qp.rb;
    }
    const RowSeq seq = {g.wj[warp], g.wn[warp], g.wr[warp], n};
    ln.ring = smem + g.ring_off + (size_t)warp * G1_DEPTH * G1_SLOT;
    ln.lane = lane;
    ln.ha = lane < width;
    ln.hb = lane + 32 < width;
    // The weights and beta are inputs that no in-flight kernel writes: the
    // first DEPTH rows of every warp go in flight before the preceding kernel
    // is waited for.
#pragma unroll
    for (int d = 0; d < G1_DEPTH; ++d) ln.fetch(seq.row(d), d);
    {  // the descriptors to shared memory, one 4-byte word per thread
        constexpr int WORDS = (int)(sizeof(G1Prob) / 4) * G1_MAX_PROBS;
        static_assert(WORDS <= G1_THREADS, "descriptor copy: one word per thread");
        if (threadIdx.x < WORDS)
            reinterpret_cast<int*>(sh.prob)[threadIdx.x] = reinterpret_cast<const int*>(g.prob)[threadIdx.x];
    }
    if (threadIdx.x < G1_MAX_PROBS) {
        const int p = threadIdx.x;
        sh.rowsum[p] = 0;
        sh.beta[p] = p < g.count && g.mode != Y_ACC ? __ldg(g.prob[p].beta) : 0.0f;
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();
    g1_stage<XM>(g, sh, smem);

    const G1Prob& q = sh.prob[pi];
    const int mode = g.mode;
    // (R = 4 with two groups per lane would not fit 64 registers; the plan
    // never chooses it)
    if (seq.R == 4)
        g1_loop<4, 1>(mode, q, sh, smem, pi, u0, seq, r0, ln);
    else if (seq.R == 2)
        width > 32 ? g1_loop<2, 2>(mode, q, sh, smem, pi, u0, seq, r0, ln)
                   : g1_loop<2, 1>(mode, q, sh, smem, pi, u0, seq, r0, ln);
    else
        width > 32 ? g1_loop<1, 2>(mode, q, sh, smem, pi, u0, seq, r0, ln)
                   : g1_loop<1, 1>(mode, q, sh, smem, pi, u0, seq, r0, ln);

    if (g.sliced) {  // every slice of every row is in: finish the sliced rows
        __syncthreads();
        for (int p = 0; p < g.count; ++p) {
            const G1Prob& qq = sh.prob[p];
            if (qq.nslice == 1) continue;
            int rr0, nn;
            g1_rows(qq, cta, ncta, rr0, nn);
            const float f = sh.fscale[p];
            const int rowsum = sh.rowsum[p];
            void* const y = qq.y;
            const int* const part = sh.part + qq.part_off;
            for (int i = threadIdx.x; i < nn; i += G1_THREADS) g1_store(mode, y, rr0 + i, part[i] - rowsum, f);
        }
    }
}

// ------------------------------------------------------------------- host

// Estimated cycles of one warp of a (problem, slice) group of n warps
// working on `rows` rows with `upl` groups per lane, and the batch size R
// that minimises it.  A batch costs a fixed latency (shared-memory loads,
// shuffle reduction, dependent arithmetic) plus its issue slots, so larger
// batches hide more latency until the rows run out.
int g1_cost(int rows, int upl, int n, int& best_r) {
    int best = 1 << 30;
    best_r = 1;
    for (int R : {4, 2, 1}) {
        if (R * upl > 4) continue;  // registers: at most four 16-byte groups of a batch per lane
        const int batches = (rows + R - 1) / R;
        const int per_warp = (batches + n - 1) / n;
        const int c = per_warp * (300 + R * (upl * 35 + 10));
        if (c < best) {
            best = c;
            best_r = R;
        }
    }
    return best;
}

// Plan the launch; false when the problem set does not suit the kernel (the
// caller then uses the general small-M kernel).
bool g1_plan(const GemvProblem* probs, int count, int x_mode, YMode mode, const DevInfo& dev, G1Params& g, int& grid,
             size_t& smem) {
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
    if (sumK > G1_MAX_SUMK || pairs > G1_WARPS) return false;
    grid = std::max(1, std::min(dev.num_sms, maxN));
    // two CTAs per SM: the shared memory of one SM (228 KB) halved, less the
    // 1 KB the hardware reserves per CTA
    const int budget = std::min(dev.max_smem_optin, 233472 / 2 - 1024);
    int off = G1_HDR, part = 0;
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
        if (q.nslice > 1) {
            q.part_off = part;
            part += (s.N + grid - 1) / grid;
        }
        g.sliced |= q.nslice > 1;
    }
    if (part > G1_PART_MAX) return false;
    g.ring_off = off;
    off += G1_WARPS * G1_DEPTH * G1_SLOT;
    if (off > budget) return false;
    // warps: one per (problem, slice) to start with, the rest to the group
    // whose slowest warp has the most work
    struct Pair {
        int p, s, rows, upl, n;
    };
    Pair pr[G1_WARPS];
    int np = 0;
    for (int i = 0; i < count; ++i) {
        const G1Prob& q = g.prob[i];
        const int U = q.K / 64;
        for (int s = 0; s < q.nslice; ++s) {
            const int width = std::min(q.slice_w, U - s * q.slice_w);
            pr[np++] = {i, s, (q.N + grid - 1) / grid, width > 32 ? 2 : 1, 1};
        }
    }
    for (int w = np; w < G1_WARPS; ++w) {
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

}  // namespace

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
    auto k = xm == X_QUANTISED ? gemv1_kernel<X_QUANTISED> : xm == X_BF16 ? gemv1_kernel<X_BF16> : gemv1_kernel<X_F32>;
    cudaError_t e = ensure_smem_optin(reinterpret_cast<const void*>(k), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(grid), dim3(G1_THREADS), smem, st, g);
}

}  // namespace bl
