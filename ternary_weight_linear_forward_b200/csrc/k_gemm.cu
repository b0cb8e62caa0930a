// k_gemm.cu -- prefill BitLinear forward (M > 64) on tcgen05 int8 tensor cores.
//
// unite.ai "Microsofts Inference Framework bringt 1-Bit grosse Sprachmodelle
// auf lokale Geraete", eq. 3 "BitLinear-Betrieb": y = W_f x_hat (beta gamma /
// Q_b).  With many tokens the ternary contraction is a dense int8 GEMM, so it
// runs on the 5th-generation tensor cores:
//
//   D[m, n] = sum_k x_q[m, k] * c[n, k]      (c = w + 1 in {0, 1, 2}, s8 x s8 -> s32)
//   acc     = D[m, n] - rowsum_m             (rowsum_m = sum_k x_q[m, k])
//
// The same kernel serves the 1-bit weights of the page's "Gewichtsbinarisierung"
// (w in {-1, +1}, 32 signs per word): their codes c = w + 1 are {0, 2}, so only
// the unpack differs.
//   y       = (float)acc * ((beta * gamma_m) / 127)
//
// Persistent kernel, one CTA per SM, output tiles of MT sub-tiles of 128 rows
// x 256 weight rows (MT = 2 from 256 tokens on, else 1), K in blocks of 128
// bytes.  Warp roles:
//   warp 0      TMA producer: x_q tile (128 MT x 128 B, 128-byte swizzle) and
//               the packed weight tile (256 rows x 8 words) per K-block, no
//               multicast;
//   warp 1      TMEM allocation and the single-thread tcgen05.mma issuer
//               (4 MMAs of K = 32 per K-block and sub-tile), tcgen05.commit to
//               free stages;
//   warps 2-5   unpack (UNPACK_WARPS = 4): packed word -> four registers of
//               codes (w >> 2s) & 0x03030303, i.e. 16 consecutive-k bytes,
//               stored as one 16-byte chunk into the 128-byte-swizzled
//               K-major operand layout;
//   warps 6..   epilogue, 4 MT warps: tcgen05.ld of the int32 accumulators (32
//               TMEM lanes per warp), rowsum correction, rescale, bf16/fp32
//               store.
// With MT = 1 two TMEM accumulators (2 x 256 columns) let the epilogue of
// tile t overlap the main loop of tile t + 1; with MT = 2 they are the two
// sub-tiles' accumulators, which share every unpacked B block (half the
// unpack and packed-weight traffic per output).  Every mbarrier wait is
// bounded.
//
// Few tiles (a few tokens: M <= 128 gives N / 256 tiles for 148 SMs) are cut
// along K: a work unit is (tile, K range) and writes its int32 tile to a
// workspace; a separate, fully parallel kernel then adds the partial tiles
// of every output (exact, so the order does not matter), subtracts the row
// sum and rescales.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace bl {

namespace {

constexpr int BM = 128;  // rows of one MMA (a sub-tile)
constexpr int BN = 256;
constexpr int BK = 128;  // bytes of K per stage
constexpr int A_SUB_BYTES = BM * BK;          // 16 KiB of x_q per sub-tile
constexpr int BC_BYTES = BN * BK;             // 32 KiB unpacked codes
constexpr int BP_BYTES = BN * (BK / 16) * 4;  // 8 KiB packed words (2-bit; 1-bit uses half)
constexpr int HDR_BYTES = 1024;
constexpr int MAX_STAGES = 4;
constexpr int UNPACK_WARPS = 4;  // measured: 4 beat 2, 8 and 16
constexpr int UNPACK_THREADS = UNPACK_WARPS * 32;
constexpr int EPI_WARP0 = 2 + UNPACK_WARPS;  // epilogue warps EPI_WARP0 .. EPI_WARP0 + 4 MT - 1

// A tile is MT sub-tiles of 128 rows on the same 256 weight rows: MT = 2
// issues two MMAs (two accumulators) per unpacked B block, halving the unpack
// and the packed-weight traffic per output; its two accumulators fill tensor
// memory, so they are not double-buffered.
template <int MT> constexpr int tile_rows() { return BM * MT; }
template <int MT> constexpr int a_bytes() { return A_SUB_BYTES * MT; }
template <int MT> constexpr int stage_bytes() { return a_bytes<MT>() + BC_BYTES + BP_BYTES; }
template <int MT> constexpr int num_stages() { return MT == 1 ? 4 : 3; }
template <int MT> constexpr int gemm_smem() { return 1024 /* alignment slack */ + HDR_BYTES + num_stages<MT>() * stage_bytes<MT>(); }
template <int MT> constexpr int gemm_threads() { return (EPI_WARP0 + 4 * MT) * 32; }
template <int MT> constexpr int acc_sets() { return MT == 1 ? 2 : 1; }
static_assert(gemm_smem<1>() <= 232448 && gemm_smem<2>() <= 232448, "GEMM stages exceed shared memory");
static_assert(num_stages<1>() <= MAX_STAGES && num_stages<2>() <= MAX_STAGES, "stage count");
static_assert(acc_sets<1>() * 1 * BN <= 512 && acc_sets<2>() * 2 * BN <= 512, "accumulators exceed TMEM");
// packed words per row and K-block: 8 of 16 trits, or 4 of 32 signs
template <int WB>
constexpr int words_per_row() { return BK * WB / 32; }
template <int WB>
constexpr int words_per_thread() { return BN * words_per_row<WB>() / UNPACK_THREADS; }
constexpr int TMEM_COLS = 512;  // two 128 x 256 int32 accumulators (double buffer, or the two sub-tiles)

constexpr uint32_t IDESC = idesc_i8(BM, BN, true, true);  // s8 x s8 -> s32, 128 x 256

struct GemmHdr {
    uint64_t full[MAX_STAGES];      // TMA bytes landed
    uint64_t unpacked[MAX_STAGES];  // codes written by the unpack threads
    uint64_t empty[MAX_STAGES];     // MMAs reading the stage finished
    uint64_t tfull[2];              // accumulator set complete
    uint64_t tempty[2];             // accumulator set drained by the 128 MT epilogue threads
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(GemmHdr) <= HDR_BYTES, "gemm header too large");

struct GemmParams {
    const float* gamma;
    const float* beta;
    const int* rowsum;
    void* y;
    int M, N, K, mode;
    int tiles_m, tiles_n, num_kb;
    int splits;     // K ranges per tile (1: no split)
    int nfull;      // units 0 .. nfull - 1 are whole tiles; each later tile is cut into `splits` K ranges
    int part_rows;  // rows of a partial tile in the workspace (min(M, tile rows))
    int* part;      // split K: [cut tiles * splits][part_rows][BN] int32 partial tiles
};

// Work unit u: whole tile u below nfull; past it, unit v = u - nfull is K
// blocks [kb0, kb1) of split v % splits of tile nfull + v / splits.  Returns
// whether the unit writes a partial tile.
__device__ __forceinline__ bool unit_range(const GemmParams& p, int u, int& t, int& kb0, int& kb1) {
    if (u < p.nfull) {
        t = u;
        kb0 = 0;
        kb1 = p.num_kb;
        return false;
    }
    const int v = u - p.nfull;
    t = p.nfull + v / p.splits;
    const int sp = v % p.splits;
    kb0 = (int)((long long)p.num_kb * sp / p.splits);
    kb1 = (int)((long long)p.num_kb * (sp + 1) / p.splits);
    return p.splits > 1;
}


__device__ __forceinline__ bool aborted(GemmHdr& h) { return *(volatile int*)&h.abort_flag != 0; }

__device__ __forceinline__ bool wait_or_abort(GemmHdr& h, uint64_t* bar, uint32_t parity) {
    if (aborted(h)) return false;
    if (!mbar_wait(bar, parity)) {
        h.abort_flag = 1;
        return false;
    }
    return true;
}

// ---------------------------------------------------------------- kernels

__global__ void __launch_bounds__(256) rowsum_kernel(const int8_t* __restrict__ x_q, int M, int K,
                                                     int* __restrict__ rowsum) {
    pdl_launch_dependents();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= M) return;
    const int4* p = reinterpret_cast<const int4*>(x_q + (long long)row * K);
    int s = 0;
    for (int g = lane; g < K / 16; g += 32) {
        int4 v = __ldg(p + g);
        s += bytesum_s8(v.x) + bytesum_s8(v.y) + bytesum_s8(v.z) + bytesum_s8(v.w);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) rowsum[row] = s;
}

// Split K: y[m, n] = (sum over the splits of the partial tiles) - rowsum_m,
// rescaled, for the outputs of the cut tiles (tiles nfull ..); four
// consecutive n per thread (one 16-byte load per split).
__global__ void __launch_bounds__(256) splitk_finish_kernel(const int* __restrict__ part, int splits, int part_rows,
                                                            int nfull, int ncut, int tiles_m, int tile_rows,
                                                            const int* __restrict__ rowsum,
                                                            const float* __restrict__ gamma,
                                                            const float* __restrict__ beta, void* __restrict__ y,
                                                            int M, int N, int mode) {
    pdl_launch_dependents();
    pdl_wait();
    const float b = mode == Y_ACC ? 0.0f : __ldg(beta);
    constexpr int NQ = BN / 4;  // quads per tile row
    const long long per_tile = (long long)part_rows * NQ;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < (long long)ncut * per_tile;
         e += (long long)gridDim.x * blockDim.x) {
        const int tt = (int)(e / per_tile);
        const int rem = (int)(e - (long long)tt * per_tile);
        const int r = rem / NQ, c = (rem % NQ) * 4;
        const int t = nfull + tt;
        const int m = (t % tiles_m) * tile_rows + r, n = (t / tiles_m) * BN + c;
        if (m >= M || n >= N) continue;
        const int4* src = reinterpret_cast<const int4*>(part + ((size_t)tt * splits * part_rows + r) * BN + c);
        int4 acc = make_int4(0, 0, 0, 0);
        for (int sp = 0; sp < splits; ++sp) {
            const int4 v = __ldcg(src + (size_t)sp * part_rows * BN / 4);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        const int rs = __ldcg(rowsum + m);
        const int a[4] = {acc.x - rs, acc.y - rs, acc.z - rs, acc.w - rs};
        const float f = mode == Y_ACC ? 0.0f : __fdiv_rn(__fmul_rn(b, __ldg(gamma + m)), 127.0f);
        for (int j = 0; j < 4 && n + j < N; ++j) {
            const long long o = (long long)m * N + n + j;
            if (mode == Y_ACC)
                reinterpret_cast<int*>(y)[o] = a[j];
            else if (mode == Y_F32)
                reinterpret_cast<float*>(y)[o] = __fmul_rn((float)a[j], f);
            else
                reinterpret_cast<uint16_t*>(y)[o] = f32_to_bf16_rn(__fmul_rn((float)a[j], f));
        }
    }
}

__device__ __forceinline__ void store_chunk(const GemmParams& p, int m, int n0, const int (&v)[32], int rs, float f,
                                            bool vec_ok) {
    const long long o = (long long)m * p.N + n0;
    const bool full = n0 + 32 <= p.N;
    if (p.mode == Y_ACC) {
        int* y = reinterpret_cast<int*>(p.y) + o;
        if (full && vec_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<int4*>(y + j) = make_int4(v[j] - rs, v[j + 1] - rs, v[j + 2] - rs, v[j + 3] - rs);
        } else {
            for (int j = 0; j < 32 && n0 + j < p.N; ++j) y[j] = v[j] - rs;
        }
    } else if (p.mode == Y_F32) {
        float* y = reinterpret_cast<float*>(p.y) + o;
        float t[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) t[j] = __fmul_rn((float)(v[j] - rs), f);
        if (full && vec_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4*>(y + j) = make_float4(t[j], t[j + 1], t[j + 2], t[j + 3]);
        } else {
            for (int j = 0; j < 32 && n0 + j < p.N; ++j) y[j] = t[j];
        }
    } else {
        uint16_t* y = reinterpret_cast<uint16_t*>(p.y) + o;
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t lo = f32_to_bf16_rn(__fmul_rn((float)(v[2 * j] - rs), f));
            const uint32_t hi = f32_to_bf16_rn(__fmul_rn((float)(v[2 * j + 1] - rs), f));
            h[j] = lo | (hi << 16);
        }
        if (full && vec_ok) {
#pragma unroll
            for (int j = 0; j < 16; j += 4) *reinterpret_cast<uint4*>(y + 2 * j) = make_uint4(h[j], h[j + 1], h[j + 2], h[j + 3]);
        } else {
            for (int j = 0; j < 32 && n0 + j < p.N; ++j) y[j] = (uint16_t)(h[j >> 1] >> ((j & 1) * 16));
        }
    }
}

template <int WB, int MT>
__global__ void __launch_bounds__(gemm_threads<MT>(), 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const GemmParams p) {
    constexpr int STAGES = num_stages<MT>();
    constexpr int STAGE_BYTES = stage_bytes<MT>();
    constexpr int A_BYTES = a_bytes<MT>();
    constexpr int SETS = acc_sets<MT>();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* base =
        smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);  // 1024-byte aligned for the swizzle
    GemmHdr& h = *reinterpret_cast<GemmHdr*>(base);
    unsigned char* stages = base + HDR_BYTES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_units = p.nfull + (p.tiles_m * p.tiles_n - p.nfull) * p.splits;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&h.full[s], 1);
            mbar_init(&h.unpacked[s], UNPACK_THREADS);
            mbar_init(&h.empty[s], 1);
        }
        for (int b = 0; b < SETS; ++b) {
            mbar_init(&h.tfull[b], 1);
            mbar_init(&h.tempty[b], 128 * MT);
        }
        h.abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) tmem_alloc(&h.tmem_base, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = h.tmem_base;
    pdl_launch_dependents();
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int it = 0;
            for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
                int t, kb0, kb1;
                unit_range(p, u, t, kb0, kb1);
                const int mb = t % p.tiles_m, nb = t / p.tiles_m;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!wait_or_abort(h, &h.empty[s], ph ^ 1)) goto done;
                    unsigned char* st = stages + (size_t)s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&h.full[s], A_BYTES + BN * words_per_row<WB>() * 4);
                    tma_load_2d(st, &tmap_a, kb * BK, mb * tile_rows<MT>(), &h.full[s]);
                    tma_load_2d(st + A_BYTES + BC_BYTES, &tmap_b, kb * words_per_row<WB>(), nb * BN, &h.full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, acc_it = 0;
            for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++acc_it) {
                int t, kb0, kb1;
                unit_range(p, u, t, kb0, kb1);
                const int b = acc_it % SETS;
                const uint32_t aph = (acc_it / SETS) & 1;
                if (!wait_or_abort(h, &h.tempty[b], aph ^ 1)) goto done;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(b * MT * BN);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!wait_or_abort(h, &h.full[s], ph)) goto done;
                    if (!wait_or_abort(h, &h.unpacked[s], ph)) goto done;
                    tc_fence_after();
                    unsigned char* st = stages + (size_t)s * STAGE_BYTES;
                    const uint64_t bdesc = sw128_desc(smem_u32(st + A_BYTES));
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {  // K = 32 bytes per MMA: advance 32 B = 2 in addr >> 4
#pragma unroll
                        for (int a = 0; a < MT; ++a)      // sub-tile a: x_q rows 128 a .., accumulator a
                            mma_i8(d_tmem + (uint32_t)(a * BN), sw128_desc(smem_u32(st + a * A_SUB_BYTES)) + 2 * k,
                                   bdesc + 2 * k, IDESC, (kb != kb0) || (k != 0));
                    }
                    mma_commit(&h.empty[s]);
                }
                mma_commit(&h.tfull[b]);
            }
        }
    } else if (warp < EPI_WARP0) {
        // ------------------------------------------------ unpack
        constexpr int WPR = words_per_row<WB>(), WPT = words_per_thread<WB>();
        const int ut = threadIdx.x - 64;  // 0 .. UNPACK_THREADS - 1
        // word w = ut + UNPACK_THREADS * i of the packed tile is row n = w / WPR,
        // word j = w % WPR.  2-bit: its 16 codes go to 16-byte chunk j ^ (n % 8)
        // of row n.  1-bit: its 32 codes go to chunks 2j and 2j + 1 (swizzled
        // the same way); dst_off holds the first, the second is found by ^ 16.
        uint32_t dst_off[WPT];
#pragma unroll
        for (int i = 0; i < WPT; ++i) {
            const int w = ut + UNPACK_THREADS * i;
            const int n = w / WPR, j = w % WPR;
            const int c = WB == 2 ? j : 2 * j;
            dst_off[i] = (uint32_t)(n * BK + ((c ^ (n & 7)) << 4));
        }
        int it = 0;
        for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
            int t, kb0, kb1;
            unit_range(p, u, t, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!wait_or_abort(h, &h.full[s], ph)) goto done;
                unsigned char* st = stages + (size_t)s * STAGE_BYTES;
                const uint32_t* bp = reinterpret_cast<const uint32_t*>(st + A_BYTES + BC_BYTES);
                const uint32_t bc = smem_u32(st + A_BYTES);
                uint32_t word[WPT];
#pragma unroll
                for (int i = 0; i < WPT; ++i) word[i] = bp[ut + UNPACK_THREADS * i];
#pragma unroll
                for (int i = 0; i < WPT; ++i) {
                    if constexpr (WB == 2) {
                        const uint32_t t0 = word[i] & 0x03030303u;
                        const uint32_t t1 = (word[i] >> 2) & 0x03030303u;
                        const uint32_t t2 = (word[i] >> 4) & 0x03030303u;
                        const uint32_t t3 = (word[i] >> 6) & 0x03030303u;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(bc + dst_off[i]), "r"(t0),
                                     "r"(t1), "r"(t2), "r"(t3)
                                     : "memory");
                    } else {
                        // sign bit of k = 32j + 4s + b at bit 8b + s -> code 2 * bit in byte b of int s
                        const uint32_t w = word[i];
                        const uint32_t t0 = (w << 1) & 0x02020202u;
                        const uint32_t t1 = w & 0x02020202u;
                        const uint32_t t2 = (w >> 1) & 0x02020202u;
                        const uint32_t t3 = (w >> 2) & 0x02020202u;
                        const uint32_t t4 = (w >> 3) & 0x02020202u;
                        const uint32_t t5 = (w >> 4) & 0x02020202u;
                        const uint32_t t6 = (w >> 5) & 0x02020202u;
                        const uint32_t t7 = (w >> 6) & 0x02020202u;
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(bc + dst_off[i]), "r"(t0),
                                     "r"(t1), "r"(t2), "r"(t3)
                                     : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(bc + (dst_off[i] ^ 16u)),
                                     "r"(t4), "r"(t5), "r"(t6), "r"(t7)
                                     : "memory");
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&h.unpacked[s]);
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lanes 32q .. 32q + 31
        const int sub = (warp - EPI_WARP0) / 4;  // sub-tile (accumulator) of this warp
        const bool vec_ok = p.mode == Y_BF16 ? (p.N % 8 == 0) : (p.N % 4 == 0);
        const float beta = p.mode == Y_ACC ? 0.0f : __ldg(p.beta);
        int acc_it = 0;
        for (int u = blockIdx.x; u < num_units; u += gridDim.x, ++acc_it) {
            int t, kb0, kb1;
            const bool cut = unit_range(p, u, t, kb0, kb1);
            const int mb = t % p.tiles_m, nb = t / p.tiles_m;
            const int b = acc_it % SETS;
            const uint32_t aph = (acc_it / SETS) & 1;
            // tcgen05.ld is warp-collective: the whole warp proceeds or leaves together
            if (!__all_sync(0xffffffffu, wait_or_abort(h, &h.tfull[b], aph))) goto done;
            tc_fence_after();
            const int r = sub * BM + q * 32 + lane;  // row of the tile
            const int m = mb * tile_rows<MT>() + r;
            int rs = 0;
            float f = 0.0f;
            if (m < p.M) {
                rs = __ldcg(p.rowsum + m);  // L2 only: written by the preceding kernel
                if (p.mode != Y_ACC) f = __fdiv_rn(__fmul_rn(beta, __ldg(p.gamma + m)), 127.0f);
            }
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)((b * MT + sub) * BN);
            if (!cut) {
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    int v[32];
                    tmem_ld32(tbase + (uint32_t)(c * 32), v);
                    const int n0 = nb * BN + c * 32;
                    if (m < p.M && n0 < p.N) store_chunk(p, m, n0, v, rs, f, vec_ok);
                }
                tc_fence_before();
                mbar_arrive(&h.tempty[b]);
                continue;
            }
            // split K: this unit's partial tile to the workspace
            int* mine = p.part + ((size_t)(u - p.nfull) * p.part_rows + r) * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                int v[32];
                tmem_ld32(tbase + (uint32_t)(c * 32), v);
                if (r < p.part_rows && m < p.M) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        __stcg(reinterpret_cast<int4*>(mine + c * 32 + j), make_int4(v[j], v[j + 1], v[j + 2], v[j + 3]));
                }
            }
            tc_fence_before();
            mbar_arrive(&h.tempty[b]);
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------- host

}  // namespace

EncodeTiled tensor_map_encoder() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(ptr);
    });
    return fn;
}

// K ranges per tile: as many as keep the units within one wave of the B200's
// 148 SMs (a fixed count, so the workspace size does not depend on the device).
constexpr int SPLIT_UNITS_TARGET = 148;

// Two sub-tiles per tile from this many tokens on (when K is not cut).
constexpr long long MT2_MIN_M = 256;

struct GemmPlan {
    int mt, tiles_m, tiles_n, num_kb, splits, nfull, part_rows;
    size_t rowsum_bytes, part_bytes;
};

GemmPlan gemm_plan(long long M, long long N, long long K, bool allow_split) {
    GemmPlan g;
    g.mt = 1;
    g.tiles_m = (int)((M + BM - 1) / BM);
    g.tiles_n = (int)((N + BN - 1) / BN);
    g.num_kb = (int)((K + BK - 1) / BK);
    const long long tiles = (long long)g.tiles_m * g.tiles_n;
    g.splits = allow_split ? (int)std::max<long long>(1, std::min<long long>(SPLIT_UNITS_TARGET / tiles, g.num_kb)) : 1;
    g.nfull = 0;
    if (g.splits == 1) {
        if (M >= MT2_MIN_M) {
            g.mt = 2;
            g.tiles_m = (int)((M + 2 * BM - 1) / (2 * BM));
        }
        g.nfull = g.tiles_m * g.tiles_n;  // every tile whole
    }
    const long long cut = (long long)g.tiles_m * g.tiles_n - g.nfull;
    g.part_rows = (int)std::min<long long>(M, (long long)g.mt * BM);
    g.rowsum_bytes = (size_t)((M * 4 + 255) / 256 * 256);
    g.part_bytes = g.splits > 1 ? (size_t)cut * g.splits * g.part_rows * BN * 4 : 0;
    return g;
}

size_t gemm_ws_bytes(long long M, long long N, long long K) {
    const GemmPlan g = gemm_plan(M, N, K, true);
    return g.rowsum_bytes + g.part_bytes;
}

cudaError_t launch_gemm(const int8_t* x_q, const float* gamma, int M, int K, const uint32_t* W_p, const float* beta,
                        int N, void* y, YMode mode, void* ws, const DevInfo& dev, cudaStream_t st, int wbits,
                        bool allow_split, bool rowsum_ready) {
    if (wbits != 1 && wbits != 2) return cudaErrorInvalidValue;
    EncodeTiled enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const GemmPlan plan = gemm_plan(M, N, K, allow_split);
    const int smem = plan.mt == 1 ? gemm_smem<1>() : gemm_smem<2>();
    if (dev.max_smem_optin < smem) return cudaErrorNotSupported;
    CUtensorMap ta, tb;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K};
        const cuuint32_t box[2] = {BK, (cuuint32_t)(plan.mt * BM)};
        const cuuint32_t estr[2] = {1, 1};
        if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(x_q), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        // row of K * wbits / 8 bytes; a box of one K-block (BK * wbits / 32 words) x BN rows
        const cuuint64_t dims[2] = {(cuuint64_t)(K * wbits / 32), (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)(K * wbits / 8)};
        const cuuint32_t box[2] = {(cuuint32_t)(BK * wbits / 32), BN};
        const cuuint32_t estr[2] = {1, 1};
        if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(W_p), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    int* rowsum = reinterpret_cast<int*>(ws);
    int* part = plan.splits > 1 ? reinterpret_cast<int*>(reinterpret_cast<char*>(ws) + plan.rowsum_bytes) : nullptr;
    cudaError_t e = cudaSuccess;
    if (!rowsum_ready) {
        e = launch_pdl(rowsum_kernel, dim3((M + 7) / 8), dim3(256), 0, st, x_q, M, K, rowsum);
        if (e != cudaSuccess) return e;
    }

    GemmParams p;
    p.gamma = gamma;
    p.beta = beta;
    p.rowsum = rowsum;
    p.y = y;
    p.M = M;
    p.N = N;
    p.K = K;
    p.mode = mode;
    p.tiles_m = plan.tiles_m;
    p.tiles_n = plan.tiles_n;
    p.num_kb = plan.num_kb;
    p.splits = plan.splits;
    p.nfull = plan.nfull;
    p.part_rows = plan.part_rows;
    p.part = part;
    const int ncut = p.tiles_m * p.tiles_n - p.nfull;
    const int units = p.nfull + ncut * p.splits;
    const int grid = std::max(1, std::min(units, dev.num_sms));
    auto kernel = plan.mt == 1 ? (wbits == 2 ? gemm_kernel<2, 1> : gemm_kernel<1, 1>)
                               : (wbits == 2 ? gemm_kernel<2, 2> : gemm_kernel<1, 2>);
    const int threads = plan.mt == 1 ? gemm_threads<1>() : gemm_threads<2>();
    e = ensure_smem_optin(reinterpret_cast<const void*>(kernel), (size_t)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kernel, dim3(grid), dim3(threads), (size_t)smem, st, ta, tb, p);
    if (e != cudaSuccess || plan.splits == 1) return e;
    const long long quads = (long long)ncut * plan.part_rows * (BN / 4);
    const int fgrid = (int)std::max<long long>(1, std::min<long long>((quads + 255) / 256, (long long)dev.num_sms * 8));
    return launch_pdl(splitk_finish_kernel, dim3(fgrid), dim3(256), 0, st, (const int*)part, plan.splits,
                      plan.part_rows, plan.nfull, ncut, plan.tiles_m, plan.mt * BM, (const int*)rowsum, gamma, beta,
                      y, M, N, (int)mode);
}

}  // namespace bl
