// k_decode_tc.cu -- decode BitLinear forward (M <= 16 tokens) on the tcgen05
// tensor cores.
//
// DataCamp blog "MatMul-free language models", section "MatMul vervangen
// door ternaire bewerkingen": with weights in {-1, 0, +1} the product is a
// ternary accumulation; unite.ai "Microsofts Inference Framework bringt 1-Bit
// grosse Sprachmodelle auf lokale Geraete", eq. 3 "BitLinear-Betrieb": the
// integer result is rescaled by beta * gamma / Q_b.  The integer arithmetic is
// that of the CUDA-core decode kernel: codes c = w + 1 in {0, 1, 2},
//
//   acc[m, n] = sum_k c[n, k] * x_hat[m, k] - sum_k x_hat[m, k]   (exact, int32)
//
// Why tensor cores at M = 1: on CUDA cores every 4 trits cost a mask and a
// half-rate dp4a, which on B200 takes longer than streaming their byte from
// HBM.  Here the CUDA cores only expand 2-bit codes to bytes and tcgen05 does
// the contraction:
//
//   * swap-AB: the MMA's M = 128 rows are weight rows (one per TMEM lane), its
//     N columns are tokens, so one token already makes a legal 128 x 16 tile;
//   * A (the codes, 4x the packed bytes) is written to tensor memory with
//     tcgen05.st and never touches shared memory, whose bandwidth would
//     otherwise bound the kernel; B (x_hat) stays in shared memory for the
//     whole K range, 128-byte-swizzled K-major;
//   * code bytes: with G = 4 column groups the unpack is one mask per 4 trits,
//     w & (0x03030303 << 2s) = 4^s c (unsigned bytes), and B holds x_hat in 4
//     columns per token, column s keeping only k with (k / 4) % 4 == s; the
//     epilogue adds D[., 4m + s] >> 2s.  Used while the MMA stays 16 wide;
//     otherwise G = 1 and the codes are (w >> 2s) & 0x03030303;
//   * when a CTA owns few rows, K is cut into S slices and row n's slice q is
//     placed in subpartition q's lanes: B holds S column blocks (one per
//     slice, zero outside it) and the epilogue adds the S partial sums, so the
//     unpack is spread over all four SM sub-partitions;
//   * the packed rows arrive by 2-D TMA (128 bytes of every row per stage,
//     128-byte swizzle so the per-lane 16-byte reads are conflict-free) into a
//     ring that starts filling as soon as the CTA starts;
//   * the unpack needs only the weights, so it starts before the kernel waits
//     for its predecessor: all six A buffers are filled while the previous
//     kernel drains, then x is quantised into B and the MMAs start.
//
// Warp roles (448 threads): warps 0-11 unpack -- three warps per TMEM
// subpartition (warp w owns lanes 32 (w % 4) ..), taking the 128-trit A
// quarters round-robin -- and build B and run the epilogue; warp 12 issues the
// TMA stream; warp 13 owns TMEM and issues the MMAs.  Every wait is bounded;
// after a timeout every role still runs its barriers, waits for its copies
// and MMAs in flight and frees TMEM.
#include <cuda.h>

#include <cstring>

#include "act_inl.cuh"
#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace bl {

namespace {

constexpr int DTC_TEAMS = 3;                                // unpack warps per TMEM subpartition
constexpr int DTC_UNPACK_WARPS = 4 * DTC_TEAMS;             // warps 0 .. 11
constexpr int DTC_UNPACK_THREADS = DTC_UNPACK_WARPS * 32;   // 384
constexpr int DTC_PRODUCER = DTC_UNPACK_WARPS;              // warp 12
constexpr int DTC_MMA = DTC_UNPACK_WARPS + 1;               // warp 13
constexpr int DTC_THREADS = (DTC_UNPACK_WARPS + 2) * 32;    // 448
constexpr int DTC_STAGE_K = 512;                            // trits per ring stage (128 bytes per row)
constexpr int DTC_QK = 128;                                 // trits per A buffer ("quarter" of a stage)
constexpr int DTC_NBUF = 6;                                 // A buffers in TMEM
constexpr int DTC_ACOLS = DTC_QK / 4;                       // 32 columns per A buffer
constexpr int DTC_DCOL = DTC_NBUF * DTC_ACOLS;              // accumulator at column 192
constexpr int DTC_TMEM_COLS = 256;
constexpr int DTC_MAX_NMMA = DTC_TMEM_COLS - DTC_DCOL;      // 64 accumulator columns
constexpr int DTC_MAX_SLOTS = 16;
constexpr int DTC_MAX_M = 16;
constexpr int DTC_HDR = 3072;
constexpr int DTC_GROUP_MAX = 8;

struct DtcHdr {
    uint64_t full[DTC_MAX_SLOTS];    // stage landed (TMA bytes)
    uint64_t empty[DTC_MAX_SLOTS];   // stage read: 4 quarters x 4 subpartitions
    uint64_t a_full[DTC_NBUF];       // A buffer written (one warp per subpartition)
    uint64_t a_empty[DTC_NBUF];      // MMAs reading the A buffer finished
    uint64_t b_ready;                // B and the per-token tables are built
    uint64_t d_full;                 // accumulator of a tile complete
    uint64_t d_empty;                // accumulator drained by the 4 epilogue warps
    uint64_t drain;                  // every MMA issued by this CTA finished
    uint32_t tmem_base;
    int abort_flag;
    int rowsum[DTC_MAX_M];           // sum of x_hat per token (zeroed at CTA start)
    int amax[DTC_MAX_M];             // max |x| per token as float bits (zeroed at CTA start)
    float gam[DTC_MAX_M];
    float xscale[DTC_MAX_M];         // 127 / gamma
    float fscale[DTC_MAX_M];
    float beta;                      // read at CTA start (a weight input)
};
static_assert(sizeof(DtcHdr) <= DTC_HDR, "decode header too large");

// One problem.  Rows are dealt to CTAs in runs of R; a CTA walks its rows in
// tiles of Rt and every tile's K range in T stages of 512 trits per slice.
struct alignas(64) DtcParams {
    CUtensorMap tmap;  // W_p as bytes [N][K/4], box {128, Rt}, 128-byte swizzle, zero fill
    const void* x;     // fp32 / bf16 activations (quantised in the prologue)
    const int8_t* x_q;
    const float* gamma;
    const int* rowsum_in;  // row sums of x_q when the quantiser wrote them (else null)
    const float* beta;
    void* y;
    int M, K, N, mode;
    int R;            // rows per CTA
    int S;            // K slices (1, 2 or 4)
    int Lfull;        // trits per slice, a multiple of 512; the last slice ends at K
    int T;            // stages per tile
    int Rt, Rt8;      // rows per tile; rounded up to 8 (ring layout)
    int ntiles;       // tiles per CTA
    int L;            // TMEM lanes used per subpartition
    int slots;        // ring slots
    int stage_bytes;  // S * Rt8 * 128
    int brow;         // B rows per 128-trit K-block (multiple of 8)
    int part_off, b_off, ring_off;  // shared-memory offsets from the 1024-aligned base
    uint32_t idesc;
};

struct DtcGroup {
    DtcParams prob[DTC_GROUP_MAX];
    int cta0[DTC_GROUP_MAX + 1];
    int count;
};

__device__ __forceinline__ bool aborted(DtcHdr& h) { return *(volatile int*)&h.abort_flag != 0; }

__device__ __forceinline__ bool wait_or_abort(DtcHdr& h, uint64_t* bar, uint32_t parity) {
    if (aborted(h)) return false;
    if (!mbar_wait(bar, parity)) {
        h.abort_flag = 1;
        return false;
    }
    return true;
}

// Warp-uniform bounded wait: the warp's tcgen05 instructions are collective.
__device__ __forceinline__ bool warp_wait(DtcHdr& h, uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, wait_or_abort(h, bar, parity));
}

__device__ __forceinline__ void unpack_sync() {
    asm volatile("bar.sync 1, %0;" ::"r"(DTC_UNPACK_THREADS) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, int4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void store_y(const DtcParams& p, int m, int n, int acc, float f) {
    const long long o = (long long)m * p.N + n;
    if (p.mode == Y_ACC) {
        reinterpret_cast<int*>(p.y)[o] = acc;
    } else {
        const float v = __fmul_rn((float)acc, f);
        if (p.mode == Y_F32)
            reinterpret_cast<float*>(p.y)[o] = v;
        else
            reinterpret_cast<uint16_t*>(p.y)[o] = f32_to_bf16_rn(v);
    }
}

// Issue ring stages [u0, u1) (unit u = tile * T + t).  Returns the number of
// stages issued in total (u1, or where a wait gave up).
__device__ __forceinline__ int produce(const DtcParams& p, DtcHdr& h, unsigned char* ring, int r0, int u0, int u1,
                                       uint64_t pol) {
    for (int u = u0; u < u1; ++u) {
        const int slot = u % p.slots;
        if (u >= p.slots && !wait_or_abort(h, &h.empty[slot], ((u / p.slots) - 1) & 1)) return u;
        const int tile = u / p.T, t = u % p.T;
        const int y0 = r0 + tile * p.Rt;
        unsigned char* dst = ring + (size_t)slot * p.stage_bytes;
        int nload = 0;
        for (int q = 0; q < p.S; ++q) nload += (q * p.Lfull + t * DTC_STAGE_K < p.K) ? 1 : 0;
        mbar_arrive_expect_tx(&h.full[slot], (uint32_t)(nload * p.Rt * 128));
        for (int q = 0; q < p.S; ++q) {
            const int k0 = q * p.Lfull + t * DTC_STAGE_K;  // slices past K leave stale bytes: B is 0 there
            if (k0 < p.K) tma_load_2d_hint(dst + (size_t)q * p.Rt8 * 128, &p.tmap, k0 / 4, y0, &h.full[slot], pol);
        }
    }
    return u1;
}

// Build B (x_hat in S column blocks of MP tokens x G groups, zero outside each
// slice, each group and for padded tokens), the per-token row sums of x_hat
// and the rescale factors.  Runs on the unpack warps after the wait for the
// preceding kernel.  Work is dealt by B row: row j = q * MP + m (slice q,
// token m) goes to warp j % 12 and its KC = 32 T chunks to the lanes, so the
// index arithmetic is shifts and masks and every row's total is one warp
// reduction plus one shared-memory atomic.  Plain int8 x_hat is copied into
// B by cp.async, all chunks in flight at once.
template <int MP, int G, int XM>
__device__ __forceinline__ void stage_b(const DtcParams& p, DtcHdr& h, int* part, unsigned char* Bs) {
    constexpr int NW = DTC_UNPACK_WARPS;
    const int ctid = threadIdx.x, lane = ctid & 31, warp = ctid >> 5;
    const size_t xrow = (size_t)p.K * (XM == X_BF16 ? 2 : XM == X_F32 ? 4 : 1);
    const char* xbase = XM == X_QUANTISED ? reinterpret_cast<const char*>(p.x_q) : reinterpret_cast<const char*>(p.x);
    // gamma and the given row sums (written by the preceding quantiser) load
    // while x_hat is staged
    float gq = 0.0f;
    int rsq = 0;
    if (XM == X_QUANTISED && ctid < MP && ctid < p.M) {
        if (p.mode != Y_ACC) gq = __ldg(p.gamma + ctid);
        if (p.rowsum_in) rsq = __ldg(p.rowsum_in + ctid);
    }
    const int rows = p.S * MP;                // B rows per K-block before the G expansion
    const int KC = p.T * (DTC_STAGE_K / 16);  // chunks per B row
    const uint32_t bs = smem_u32(Bs);
    // chunk kc of row j: byte offset in B (G = 1), and whether it holds data
    auto slot = [&](int j, int kc) -> uint32_t {
        return (uint32_t)((kc >> 3) * p.brow * 128 + j * 128 + (((kc & 7) ^ (j & 7)) << 4));
    };
    if (XM != X_QUANTISED) {
        // pass 1: max |x| of every token (exact, order-free)
        for (int j = warp; j < rows; j += NW) {
            const int q = j / MP, m = j % MP;
            unsigned a = 0u;
            if (m < p.M) {
                const int ls = min(p.Lfull, p.K - q * p.Lfull);
                const char* xr = xbase + (size_t)m * xrow;
#pragma unroll 2
                for (int kc = lane; kc * 16 < ls; kc += 32) {
                    XChunk<XM> c;
                    ld_chunk<XM>(xr, (q * p.Lfull + kc * 16) / 16, c);
                    a = chunk_absmax<XM>(c, a);
                }
            }
            a = __reduce_max_sync(0xffffffffu, a);
            if (lane == 0 && a != 0u) atomicMax(&h.amax[m], (int)a);
        }
        unpack_sync();
        if (ctid < MP) {
            const float g = fmaxf(__int_as_float(h.amax[ctid]), 1e-5f);
            h.gam[ctid] = g;
            h.xscale[ctid] = __fdiv_rn(127.0f, g);
        }
        unpack_sync();
    }
    for (int i = ctid; i < p.Rt * MP; i += DTC_UNPACK_THREADS) part[i] = 0;
    // pass 2: 16-byte chunks of x_hat into B.  Row (q * MP + m) * G + s of
    // K-block kb holds group s of x_hat[m, q * Lfull + 128 kb ...]; chunk c of
    // a row sits at c ^ (row % 8).
    if constexpr (XM == X_QUANTISED && G == 1) {
        for (int j = warp; j < rows; j += NW) {
            const int q = j / MP, m = j % MP;
            const int ls = m < p.M ? min(p.Lfull, p.K - q * p.Lfull) : 0;
            const int8_t* xr = p.x_q + (size_t)m * p.K + q * p.Lfull;
            for (int kc = lane; kc < KC; kc += 32) {
                if (kc * 16 < ls)
                    cp_async16(bs + slot(j, kc), xr + kc * 16);
                else
                    sts128(bs + slot(j, kc), make_int4(0, 0, 0, 0));
            }
        }
        cp_async_wait_all();
        for (int j = warp; j < rows && !p.rowsum_in; j += NW) {
            const int m = j % MP;
            int rs = 0;
            for (int kc = lane; kc < KC; kc += 32) {
                const uint4 v = lds128(bs + slot(j, kc));
                rs += bytesum_s8((int)v.x) + bytesum_s8((int)v.y) + bytesum_s8((int)v.z) + bytesum_s8((int)v.w);
            }
            rs = __reduce_add_sync(0xffffffffu, rs);
            if (lane == 0 && rs != 0) atomicAdd(&h.rowsum[m], rs);
        }
    } else {
        for (int j = warp; j < rows; j += NW) {
            const int q = j / MP, m = j % MP;
            const int ls = m < p.M ? min(p.Lfull, p.K - q * p.Lfull) : 0;
            const char* xr = xbase + (size_t)m * xrow;
            const float sc = XM == X_QUANTISED ? 0.0f : h.xscale[m];
            int rs = 0;
#pragma unroll 2
            for (int kc = lane; kc < KC; kc += 32) {
                int4 v = make_int4(0, 0, 0, 0);
                if (kc * 16 < ls) {
                    XChunk<XM> c;
                    ld_chunk<XM>(xr, (q * p.Lfull + kc * 16) / 16, c);
                    v = chunk_codes<XM>(c, sc);
                    rs += bytesum_s8(v.x) + bytesum_s8(v.y) + bytesum_s8(v.z) + bytesum_s8(v.w);
                }
                if (G == 1) {
                    sts128(bs + slot(j, kc), v);
                } else {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int4 vg =
                            make_int4(g == 0 ? v.x : 0, g == 1 ? v.y : 0, g == 2 ? v.z : 0, g == 3 ? v.w : 0);
                        sts128(bs + slot(j * 4 + g, kc), vg);
                    }
                }
            }
            rs = __reduce_add_sync(0xffffffffu, rs);
            if (lane == 0 && rs != 0) atomicAdd(&h.rowsum[m], rs);
        }
    }
    fence_proxy_async_smem();  // B is read by the tensor cores (async proxy)
    unpack_sync();
    if (ctid < MP) {
        const int m = ctid;
        float f = 0.0f;
        if (p.mode != Y_ACC && m < p.M) {
            const float g = XM == X_QUANTISED ? gq : h.gam[m];
            f = __fdiv_rn(__fmul_rn(h.beta, g), 127.0f);
        }
        h.fscale[m] = f;
        if (XM == X_QUANTISED && p.rowsum_in && m < p.M) h.rowsum[m] = rsq;
    }
    unpack_sync();
    if (ctid == 0) mbar_arrive(&h.b_ready);
}

// MMA issuer (one thread): 4 MMAs of K = 32 per A buffer, accumulator at
// column DTC_DCOL, fresh for every tile.
__device__ __forceinline__ void mma_loop(const DtcParams& p, DtcHdr& h, unsigned char* Bs, uint32_t tmem) {
    if (!wait_or_abort(h, &h.b_ready, 0)) return;
    tc_fence_after();
    const uint32_t bbase = smem_u32(Bs);
    const uint32_t kb_bytes = (uint32_t)p.brow * 128;
    const int QT = 4 * p.T;  // quarters per tile
    int u4 = 0;
    for (int tile = 0; tile < p.ntiles; ++tile) {
        if (tile > 0) {
            if (!wait_or_abort(h, &h.d_empty, (tile - 1) & 1)) return;
            tc_fence_after();
        }
        for (int kq = 0; kq < QT; ++kq, ++u4) {
            const int b = u4 % DTC_NBUF;
            if (!wait_or_abort(h, &h.a_full[b], (u4 / DTC_NBUF) & 1)) return;
            tc_fence_after();
            const uint64_t bdesc = sw128_desc(bbase + (uint32_t)kq * kb_bytes);  // B K-block kq of the tile
#pragma unroll
            for (int kk = 0; kk < DTC_QK / 32; ++kk)
                mma_i8_ts(tmem + DTC_DCOL, tmem + (uint32_t)(b * DTC_ACOLS + kk * 8), bdesc + (uint64_t)(2 * kk),
                          p.idesc, (kq | kk) != 0);
            mma_commit(&h.a_empty[b]);
        }
        mma_commit(&h.d_full);
    }
}

// One A quarter (128 trits of every row of the tile) from the ring into TMEM
// buffer u4 % DTC_NBUF.  Returns whether the stage was there (for its release).
template <int G>
__device__ __forceinline__ void unpack_quarter(const DtcParams& p, DtcHdr& h, uint32_t ring_s, uint32_t row_off,
                                               uint32_t key, uint32_t t_lane, int tile, int kq, int u4) {
    const int lane = threadIdx.x & 31;
    const int t = kq >> 2, qq = kq & 3;
    const int u = tile * p.T + t;
    const int slot = u % p.slots;
    const int b = u4 % DTC_NBUF;
    bool ok = warp_wait(h, &h.full[slot], (u / p.slots) & 1);
    if (u4 >= DTC_NBUF) ok = warp_wait(h, &h.a_empty[b], ((u4 / DTC_NBUF) - 1) & 1) && ok;
    if (ok) {
        tc_fence_after();
        const uint32_t rowaddr = ring_s + (uint32_t)slot * p.stage_bytes + row_off;
        const uint4 w0 = lds128(rowaddr + (((uint32_t)(2 * qq) ^ key) << 4));
        const uint4 w1 = lds128(rowaddr + (((uint32_t)(2 * qq + 1) ^ key) << 4));
        const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (G == 4) {  // 4^s * c: one mask per 4 trits
                v[4 * j + 0] = wd[j] & 0x03030303u;
                v[4 * j + 1] = wd[j] & 0x0C0C0C0Cu;
                v[4 * j + 2] = wd[j] & 0x30303030u;
                v[4 * j + 3] = wd[j] & 0xC0C0C0C0u;
            } else {       // c
                v[4 * j + 0] = wd[j] & 0x03030303u;
                v[4 * j + 1] = (wd[j] >> 2) & 0x03030303u;
                v[4 * j + 2] = (wd[j] >> 4) & 0x03030303u;
                v[4 * j + 3] = (wd[j] >> 6) & 0x03030303u;
            }
        }
        tmem_st32(t_lane + (uint32_t)(b * DTC_ACOLS), v);
        tmem_wait_st();
        tc_fence_before();
    }
    __syncwarp();
    if (ok && lane == 0) {
        mbar_arrive(&h.a_full[b]);
        mbar_arrive(&h.empty[slot]);
    }
}

// Unpack warps: A quarters round-robin over the three teams of a subpartition;
// B is built once the first DTC_NBUF quarters are in TMEM; per tile, the
// epilogue.
template <int MP, int G, int XM>
__device__ __forceinline__ void unpack_loop(const DtcParams& p, DtcHdr& h, int* part, unsigned char* Bs,
                                            unsigned char* ring, uint32_t tmem, int r0, int nrows) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sp = warp & 3, tw = warp >> 2;  // TMEM subpartition; team inside it
    const int P = 4 / p.S;                    // subpartitions per slice
    const int q = sp / P;
    const int n = (sp % P) * p.L + lane;      // row of the tile held in this lane
    const bool valid = lane < p.L && n < p.Rt;
    const int nr = valid ? n : 0;             // idle lanes read row 0; their D rows are unused
    const uint32_t row_off = (uint32_t)((q * p.Rt8 + nr) * 128);
    const uint32_t key = (uint32_t)(nr & 7);
    const uint32_t ring_s = smem_u32(ring);
    const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
    const int QT = 4 * p.T;
    bool staged = false;
    for (int tile = 0; tile < p.ntiles; ++tile) {
        for (int kq = tw; kq < QT; kq += DTC_TEAMS) {
            const int u4 = tile * QT + kq;
            if (!staged && u4 >= DTC_NBUF) {  // A buffers all written once: now x and B
                pdl_wait();
                stage_b<MP, G, XM>(p, h, part, Bs);
                staged = true;
            }
            unpack_quarter<G>(p, h, ring_s, row_off, key, t_lane, tile, kq, u4);
        }
        if (!staged) {
            pdl_wait();
            stage_b<MP, G, XM>(p, h, part, Bs);
            staged = true;
        }
        // ---- epilogue of this tile: slice partial sums -> part[n][m]
        if (tw == 0) {
            if (warp_wait(h, &h.d_full, tile & 1)) {
                tc_fence_after();
                int d[MP * G];
                tmem_ld_n<MP * G>(t_lane + (uint32_t)(DTC_DCOL + q * MP * G), d);
                if (valid) {
#pragma unroll
                    for (int m = 0; m < MP; ++m) {
                        int a = d[m * G];
                        if (G == 4) a += (d[m * 4 + 1] >> 2) + (d[m * 4 + 2] >> 4) + (d[m * 4 + 3] >> 6);
                        if (m < p.M) atomicAdd(&part[n * MP + m], a);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0 && tile + 1 < p.ntiles) mbar_arrive(&h.d_empty);
            }
        }
        unpack_sync();
        const int tr0 = tile * p.Rt;
        const int tn = max(0, min(p.Rt, nrows - tr0));
        for (int i = threadIdx.x; i < p.M * p.Rt; i += DTC_UNPACK_THREADS) {
            const int m = i / p.Rt, nn = i - m * p.Rt;
            if (nn < tn && !aborted(h)) store_y(p, m, r0 + tr0 + nn, part[nn * MP + m] - h.rowsum[m], h.fscale[m]);
            part[nn * MP + m] = 0;
        }
        unpack_sync();
    }
}

template <int MP, int G, int XM>
__device__ __forceinline__ void dtc_body(const DtcParams& p, int cta) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    DtcHdr& h = *reinterpret_cast<DtcHdr*>(base);
    int* part = reinterpret_cast<int*>(base + p.part_off);
    unsigned char* Bs = base + p.b_off;
    unsigned char* ring = base + p.ring_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = cta * p.R;
    const int nrows = min(p.R, p.N - r0);
    const int units = p.ntiles * p.T;
    const uint64_t pol = policy_evict_first();

    // Thread 0 sets up the barriers and puts the first stage in flight; the
    // producer warp streams the rest.  The weights are not written by a
    // preceding kernel, so they are read before waiting for it.
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.slots; ++s) {
            mbar_init(&h.full[s], 1);
            mbar_init(&h.empty[s], 16);
        }
        for (int b = 0; b < DTC_NBUF; ++b) {
            mbar_init(&h.a_full[b], 4);
            mbar_init(&h.a_empty[b], 1);
        }
        mbar_init(&h.b_ready, 1);
        mbar_init(&h.d_full, 1);
        mbar_init(&h.d_empty, 4);
        mbar_init(&h.drain, 1);
        h.abort_flag = 0;
        for (int m = 0; m < DTC_MAX_M; ++m) h.rowsum[m] = h.amax[m] = 0;
        h.beta = p.mode == Y_ACC ? 0.0f : __ldg(p.beta);
        fence_mbar_init();
        prefetch_tmap(&p.tmap);
        produce(p, h, ring, r0, 0, 1, pol);
    }
    if (warp == DTC_MMA) tmem_alloc(&h.tmem_base, DTC_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = h.tmem_base;
    pdl_launch_dependents();

    if (warp == DTC_PRODUCER) {
        if (lane == 0) {
            const int issued = units > 1 ? produce(p, h, ring, r0, 1, units, pol) : 1;
            // no copy may still be landing when the CTA exits
            for (int u = max(0, issued - p.slots); u < issued; ++u) mbar_wait(&h.full[u % p.slots], (u / p.slots) & 1);
        }
        __syncwarp();
    } else if (warp == DTC_MMA) {
        if (lane == 0) {
            mma_loop(p, h, Bs, tmem);
            mma_commit(&h.drain);  // tracks every MMA issued above
            mbar_wait(&h.drain, 0);
        }
        __syncwarp();
    } else {
        unpack_loop<MP, G, XM>(p, h, part, Bs, ring, tmem, r0, nrows);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == DTC_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, DTC_TMEM_COLS);
    }
}

template <int MP, int G, int XM>
__global__ void __launch_bounds__(DTC_THREADS, 2) decode_tc_kernel(const __grid_constant__ DtcGroup g) {
    int i = 0;
    while (i + 1 < g.count && (int)blockIdx.x >= g.cta0[i + 1]) ++i;
    dtc_body<MP, G, XM>(g.prob[i], (int)blockIdx.x - g.cta0[i]);
}

// ------------------------------------------------------------------- host

using DtcKernel = void (*)(const DtcGroup);

template <int XM>
DtcKernel dtc_kernel_for(int mp, int g) {
    if (g == 4) {
        switch (mp) {
            case 1: return decode_tc_kernel<1, 4, XM>;
            case 2: return decode_tc_kernel<2, 4, XM>;
            default: return decode_tc_kernel<4, 4, XM>;
        }
    }
    switch (mp) {
        case 1: return decode_tc_kernel<1, 1, XM>;
        case 2: return decode_tc_kernel<2, 1, XM>;
        case 4: return decode_tc_kernel<4, 1, XM>;
        case 8: return decode_tc_kernel<8, 1, XM>;
        default: return decode_tc_kernel<16, 1, XM>;
    }
}

int pow2_at_least(int v) {
    int r = 1;
    while (r < v) r <<= 1;
    return r;
}

int round_up(int v, int a) { return (v + a - 1) / a * a; }

// K slices and row tiles for M tokens (padded to mp) and R rows per CTA.  A
// tile holds up to 128 / S rows, each split into S K-slices placed in
// different TMEM subpartitions; every tile costs Lfull / 32 MMAs, whatever
// the number of its rows, so the split with the fewest tiles x Lfull wins
// (ties: fewer tiles).
bool dtc_split(int mp, int K, int R, int& S, int& Lfull, int& ntiles, int& Rt) {
    long long best = -1;
    for (int s : {1, 2, 4}) {
        if (s * mp > DTC_MAX_NMMA) continue;
        const int lf = round_up((K + s - 1) / s, DTC_STAGE_K);
        if ((s - 1) * lf >= K) continue;  // every slice must hold data
        const int nt = (R + 128 / s - 1) / (128 / s);
        const long long cost = (long long)nt * lf;
        if (best < 0 || cost < best) {
            best = cost;
            S = s;
            Lfull = lf;
            ntiles = nt;
            Rt = (R + nt - 1) / nt;
        }
    }
    return best >= 0;
}

// Shape and shared-memory layout of one problem with G column groups for a
// CTA budget of `budget` bytes of dynamic shared memory; false when it does
// not fit.
bool dtc_layout(DtcParams& p, int G, int M, int K, int N, const DevInfo& dev, int budget, int& grid, size_t& smem) {
    if (M < 1 || M > DTC_MAX_M || K < 64 || K % 64 || N < 1) return false;
    const int mp = pow2_at_least(M);
    const int R = (N + dev.num_sms - 1) / dev.num_sms;
    grid = (N + R - 1) / R;
    int S, Lfull, ntiles, Rt;
    if (!dtc_split(mp, K, R, S, Lfull, ntiles, Rt)) return false;
    if (G == 4 && 4 * S * mp > 16) return false;  // column groups only while the MMA stays 16 wide
    p.M = M;
    p.K = K;
    p.N = N;
    p.R = R;
    p.S = S;
    p.Lfull = Lfull;
    p.T = Lfull / DTC_STAGE_K;
    p.Rt = Rt;
    p.Rt8 = round_up(Rt, 8);
    p.ntiles = ntiles;
    p.L = (Rt + (4 / S) - 1) / (4 / S);
    p.stage_bytes = S * p.Rt8 * 128;
    p.brow = round_up(S * mp * G, 8);
    const int nmma = std::max(16, round_up(S * mp * G, 16));
    if (nmma > DTC_MAX_NMMA || p.L > 32) return false;
    p.idesc = idesc_i8(128, nmma, /*a_signed=*/false, /*b_signed=*/true);
    p.part_off = DTC_HDR;
    p.b_off = round_up(DTC_HDR + Rt * mp * 4, 1024);
    // rows brow .. nmma - 1 of the last K-block read up to 1 KiB past B
    const int b_bytes = p.T * (DTC_STAGE_K / DTC_QK) * p.brow * 128 + (nmma > p.brow ? 1024 : 0);
    p.ring_off = p.b_off + b_bytes;
    const int avail = budget - 1024 /* alignment slack */ - p.ring_off;
    const int units = ntiles * p.T;
    const int slots = std::min(std::min(units, DTC_MAX_SLOTS), avail / p.stage_bytes);
    if (slots < std::min(units, 2)) return false;
    p.slots = slots;
    smem = (size_t)(1024 + p.ring_off + slots * p.stage_bytes);
    return true;
}

// G = 4 where it applies, else G = 1; `G` in: 0 (choose) or the G to use.
bool dtc_configure(DtcParams& p, int& G, int M, int K, int N, const DevInfo& dev, int budget, int& grid,
                   size_t& smem) {
    if (G != 1 && dtc_layout(p, 4, M, K, N, dev, budget, grid, smem)) {
        G = 4;
        return true;
    }
    G = 1;
    return dtc_layout(p, 1, M, K, N, dev, budget, grid, smem);
}

bool dtc_encode(DtcParams& p, const uint32_t* W_p) {
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)(p.K / 4), (cuuint64_t)p.N};
    const cuuint64_t strides[1] = {(cuuint64_t)(p.K / 4)};
    const cuuint32_t box[2] = {128, (cuuint32_t)p.Rt};
    const cuuint32_t estr[2] = {1, 1};
    return enc(&p.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(W_p), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int group_budget(const DevInfo& dev, int count) { return (dev.max_smem_optin - 1024) / std::max(2, count); }

}  // namespace

int decode_tc_max_m() { return DTC_MAX_M; }

bool decode_tc_supported(int M, int K, int N, int count, const DevInfo& dev) {
    DtcParams p = {};
    int G = 0, grid;
    size_t smem;
    return count >= 1 && count <= DTC_GROUP_MAX &&
           dtc_configure(p, G, M, K, N, dev, group_budget(dev, count), grid, smem);
}

int decode_tc_row_tiles(int M, int K, int N, const DevInfo& dev) {
    DtcParams p = {};
    int G = 0, grid;
    size_t smem;
    return dtc_configure(p, G, M, K, N, dev, group_budget(dev, 1), grid, smem) ? p.ntiles : 0;
}

cudaError_t launch_decode_tc(const GemvProblem* probs, int count, int M, int x_dtype, YMode mode, const DevInfo& dev,
                             cudaStream_t st) {
    // x_dtype: 0 fp32, 1 bf16 (quantiser fused), 2 int8 x_q with gamma
    if (count < 1 || count > DTC_GROUP_MAX) return cudaErrorInvalidValue;
    const int xm = x_dtype == 2 ? X_QUANTISED : x_dtype == 1 ? X_BF16 : X_F32;
    // the problems of a group share each SM; at least two CTAs fit an SM so the
    // next kernel can start its stream under this one's tail
    int budget = group_budget(dev, count);
    if (count == 1) {
        // A lone problem whose ring cannot hold all of its stages at two CTAs
        // per SM takes the whole SM instead: its weight stream is then never
        // throttled by slot reuse (measured at M = 16, N = 11008: the stream
        // of 2 slots ran 3 us per stage behind the tensor cores).
        DtcParams t = {};
        int gt = 0, grid;
        size_t sm;
        const int full = dev.max_smem_optin - 1024;
        if (dtc_configure(t, gt, M, probs[0].K, probs[0].N, dev, budget, grid, sm) && t.slots < t.ntiles * t.T &&
            dtc_configure(t, gt, M, probs[0].K, probs[0].N, dev, full, grid, sm))
            budget = full;
    }
    DtcGroup g;
    memset(&g, 0, sizeof(g));
    g.count = count;
    // one kernel serves the group: G = 4 only if every problem takes it
    int G = 0;
    for (int i = 0; i < count; ++i) {
        int gi = G, grid;
        size_t sm;
        if (!dtc_configure(g.prob[i], gi, M, probs[i].K, probs[i].N, dev, budget, grid, sm))
            return cudaErrorInvalidValue;
        if (gi == 1) G = 1;
    }
    if (G == 0) G = 4;
    size_t smem = 0;
    int cta = 0;
    for (int i = 0; i < count; ++i) {
        const GemvProblem& q = probs[i];
        DtcParams& p = g.prob[i];
        int grid;
        size_t sm;
        if (!dtc_layout(p, G, M, q.K, q.N, dev, budget, grid, sm)) return cudaErrorInvalidValue;
        if (!dtc_encode(p, q.W_p)) return cudaErrorInvalidValue;
        if (xm == X_QUANTISED) {
            p.x_q = static_cast<const int8_t*>(q.x);
            p.gamma = q.gamma;
            p.rowsum_in = q.rowsum;
        } else {
            p.x = q.x;
        }
        p.beta = q.beta;
        p.y = q.y;
        p.mode = mode;
        g.cta0[i] = cta;
        cta += grid;
        smem = std::max(smem, sm);
    }
    g.cta0[count] = cta;
    const int mp = pow2_at_least(M);
    DtcKernel k = xm == X_QUANTISED ? dtc_kernel_for<X_QUANTISED>(mp, G)
                  : xm == X_BF16    ? dtc_kernel_for<X_BF16>(mp, G)
                                    : dtc_kernel_for<X_F32>(mp, G);
    cudaError_t e = ensure_smem_optin(reinterpret_cast<const void*>(k), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k, dim3(cta), dim3(DTC_THREADS), smem, st, g);
}

}  // namespace bl
