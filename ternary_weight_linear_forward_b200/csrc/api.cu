// api.cu -- the extern "C" boundary of libbitlinear: host-side validation,
// device checks and dispatch.  Every entry point is declared, with its
// defining passage, in include/bitlinear.h.
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

namespace bl {

__device__ int g_dev_error = 0;

namespace {

constexpr int MAX_DEVICES = 64;

struct DevState {
    std::once_flag once;
    bool ok = false;
    DevInfo info = {0, 0};
};
DevState g_dev[MAX_DEVICES];

// Current device, checked once per device: present and compute capability 10.x.
bl_status current_device(DevInfo& out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        cudaGetLastError();
        return BL_ERR_DEVICE;
    }
    DevState& s = g_dev[dev];
    std::call_once(s.once, [&]() {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
            cudaGetLastError();
            return;
        }
        if (prop.major != 10) return;
        s.info.num_sms = prop.multiProcessorCount;
        s.info.max_smem_optin = (int)prop.sharedMemPerBlockOptin;
        s.ok = true;
    });
    if (!s.ok) return BL_ERR_DEVICE;
    out = s.info;
    return BL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

bl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BL_OK : BL_ERR_CUDA; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// N, K limits shared by the weight calls
bl_status check_nk(int64_t N, int64_t K, int64_t k_mult) {
    if (N < 1 || K < 1 || K % k_mult != 0 || K > BL_MAX_K || N > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    return BL_OK;
}

// wbits: 2 for packed trits (K % 64 == 0), 1 for packed signs (K % 128 == 0)
bl_status check_forward(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, const uint32_t* W_p,
                        const float* beta, int64_t N, const void* y, size_t y_elem, int wbits = 2) {
    if (!x_q || !W_p || !y || (y_elem != 4 && (!gamma || !beta))) return BL_ERR_NULL;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(N, K, wbits == 2 ? 64 : 128);
    if (s) return s;
    if (!aligned16(x_q) || !aligned16(W_p) || !aligned16(y) || (gamma && !aligned16(gamma)) ||
        (beta && !aligned16(beta)))
        return BL_ERR_ALIGN;
    const size_t ybytes = (size_t)M * N * y_elem;
    if (overlap(y, ybytes, x_q, (size_t)M * K) || overlap(y, ybytes, W_p, (size_t)N * K * wbits / 8) ||
        overlap(y, ybytes, gamma, gamma ? (size_t)M * 4 : 0) || overlap(y, ybytes, beta, beta ? 4 : 0))
        return BL_ERR_ALIAS;
    return BL_OK;
}

constexpr int GEMV_MAX_M = 64;

std::atomic<int> g_engine{BL_ENGINE_AUTO};
std::atomic<int> g_expire_next_wait{0};

// Which kernel runs a problem set of M tokens.  Measured on B200 (4096 x 4096
// and 4096 x 11008, x_q given): a kind::i8 tcgen05 MMA costs about the same
// ~186 cycles for any N <= 256, so with few tokens dp4a on CUDA cores streams
// the weights fastest (M <= 4); for 5 <= M <= 16 the swap-AB decode kernel
// (7.8-22 us) beats the GEMM (~21 us, one 128-row tile and a row-sum launch)
// and the CUDA cores (17-105 us); beyond that the GEMM wins (M = 64: 23-26 us
// against 193-482 us on CUDA cores).
constexpr int AUTO_CUDA_MAX_M = 4;
// Above this many tokens, one problem whose CTAs hold more rows than one
// 128-lane tile goes to the split-K GEMM: the swap-AB kernel then issues its
// MMAs tile after tile at 16 x S columns each, and measured slower (K = 4096,
// N = 11008: ~19 us at M = 16 against 16.4 us for the GEMM, while at M = 6-8
// the swap-AB kernel takes 15.5 us; at N = 4096, one tile, 9.6 us against
// ~12 us for the GEMM).
constexpr int AUTO_TC_ONE_TILE_ABOVE_M = 8;

DecodePath pick_path(int M, const GemvProblem* probs, int count, const DevInfo& dev) {
    if (M > GEMV_MAX_M) return PATH_GEMM;
    const int engine = g_engine.load(std::memory_order_relaxed);
    if (engine == BL_ENGINE_CUDA_CORES || engine == BL_ENGINE_CUDA_CORES_GENERAL) return PATH_CUDA;
    const bool tc_first = engine == BL_ENGINE_TENSOR_CORES || M > AUTO_CUDA_MAX_M;
    if (tc_first && M <= decode_tc_max_m()) {
        bool ok = true;
        for (int i = 0; i < count; ++i) ok = ok && decode_tc_supported(M, probs[i].K, probs[i].N, count, dev);
        if (ok && engine == BL_ENGINE_AUTO && count == 1 && M > AUTO_TC_ONE_TILE_ABOVE_M &&
            decode_tc_row_tiles(M, probs[0].K, probs[0].N, dev) > 1)
            return PATH_GEMM;
        if (ok) return PATH_TC;
    }
    return M <= AUTO_CUDA_MAX_M ? PATH_CUDA : PATH_GEMM;
}

// rowsum_ready: the quantiser has written the row sums of x_q at the start
// of ws (read by the tensor-core paths).
bl_status run_forward(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, const uint32_t* W_p,
                      const float* beta, int64_t N, void* y, YMode mode, void* ws, size_t ws_bytes, void* stream,
                      bool rowsum_ready = false) {
    const size_t need = bitlinear_forward_workspace(M, N, K);
    if (need && (!ws || ws_bytes < need)) return BL_ERR_WORKSPACE;
    if (need && !aligned16(ws)) return BL_ERR_ALIGN;
    DevInfo dev;
    bl_status s = current_device(dev);
    if (s) return s;
    cudaError_t e;
    GemvProblem prob = {x_q, gamma, W_p, beta, y, (int)K, (int)N};
    const DecodePath path = pick_path((int)M, &prob, 1, dev);
    if (rowsum_ready) prob.rowsum = reinterpret_cast<const int*>(ws);
    if (path == PATH_TC)
        e = launch_decode_tc(&prob, 1, (int)M, BL_I8, mode, dev, as_stream(stream));
    else if (path == PATH_CUDA)
        e = launch_decode_cuda(&prob, 1, (int)M, BL_I8, mode, dev, as_stream(stream));
    else
        e = launch_gemm(x_q, gamma, (int)M, (int)K, W_p, beta, (int)N, y, mode, ws, dev, as_stream(stream), 2, true,
                        rowsum_ready);
    return from_cuda(e);
}

// 1-bit weights: the CUDA-core GEMV for a few tokens whose x_hat fits its
// shared memory, the tensor-core GEMM otherwise.
bool bits_on_gemv(int64_t M, int64_t K) { return M <= AUTO_CUDA_MAX_M && gemv_bits_ok(M, K); }

size_t forward_bits_ws(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || K < 1 || bits_on_gemv(M, K)) return 0;
    return gemm_ws_bytes(M, N, K);
}

bl_status run_forward_bits(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, const uint32_t* W_p,
                           const float* beta, int64_t N, void* y, YMode mode, void* ws, size_t ws_bytes,
                           void* stream) {
    const size_t need = forward_bits_ws(M, N, K);
    if (need && (!ws || ws_bytes < need)) return BL_ERR_WORKSPACE;
    if (need && !aligned16(ws)) return BL_ERR_ALIGN;
    DevInfo dev;
    bl_status s = current_device(dev);
    if (s) return s;
    cudaError_t e;
    if (bits_on_gemv(M, K))
        e = launch_gemv_bits(x_q, BL_I8, gamma, (int)M, (int)K, W_p, beta, (int)N, y, mode, dev, as_stream(stream));
    else
        e = launch_gemm(x_q, gamma, (int)M, (int)K, W_p, beta, (int)N, y, mode, ws, dev, as_stream(stream), 1);
    return from_cuda(e);
}

// ---- group quantisation along K (G contiguous groups of K / G channels) ----

bool groups_ok(int64_t K, int64_t G) { return G >= 1 && G <= BL_MAX_GROUPS && K % (64 * G) == 0; }

// int32 elements between the starts of two groups' [M, N] accumulator blocks
// (rounded up so that every block starts 16-byte aligned)
long long group_acc_stride(int64_t M, int64_t N) { return (M * N + 3) / 4 * 4; }

size_t round256z(size_t n) { return (n + 255) / 256 * 256; }

// acc[g] (at acc + g * stride) = sum over group g of W_t x_q, for every group
bl_status run_grouped_acc(const int8_t* x_q, int64_t M, int64_t K, int64_t G, const uint32_t* W_p, int64_t N,
                          int* acc, long long stride, void* fws, size_t fws_bytes, const DevInfo& dev, void* stream) {
    const int64_t Kg = K / G;
    if (M <= AUTO_CUDA_MAX_M && gemv_fused_quant_ok(M, Kg)) {
        // every group is one problem of a single launch
        GemvProblem probs[BL_MAX_GROUPS];
        for (int64_t g = 0; g < G; ++g)
            probs[g] = {x_q + g * M * Kg, nullptr, W_p + g * N * (Kg / 16), nullptr, acc + g * stride, (int)Kg, (int)N};
        const cudaError_t e = pick_path((int)M, probs, (int)G, dev) == PATH_TC
                                  ? launch_decode_tc(probs, (int)G, (int)M, BL_I8, Y_ACC, dev, as_stream(stream))
                                  : launch_decode_cuda(probs, (int)G, (int)M, BL_I8, Y_ACC, dev, as_stream(stream));
        return from_cuda(e);
    }
    for (int64_t g = 0; g < G; ++g) {
        bl_status s = run_forward(x_q + g * M * Kg, nullptr, M, Kg, W_p + g * N * (Kg / 16), nullptr, N,
                                  acc + g * stride, Y_ACC, fws, fws_bytes, stream);
        if (s) return s;
    }
    return BL_OK;
}

size_t grouped_ws(int64_t M, int64_t N, int64_t K, int64_t G) {
    if (M < 1 || N < 1 || !groups_ok(K, G)) return 0;
    return round256z((size_t)group_acc_stride(M, N) * G * 4) + round256z(bitlinear_forward_workspace(M, N, K / G));
}

}  // namespace

DecodePath decode_path(int M, const GemvProblem* probs, int count, const DevInfo& dev) {
    return pick_path(M, probs, count, dev);
}

bool take_wait_expiry_request() { return g_expire_next_wait.exchange(0, std::memory_order_relaxed) != 0; }

// Whether the automatic engine runs one token on the streaming one-token
// kernel (else on the general small-M kernel); BL_ENGINE_CUDA_CORES always
// does where the kernel applies.
constexpr bool AUTO_ONE_TOKEN_STREAMING = false;

cudaError_t launch_decode_cuda(const GemvProblem* probs, int count, int M, int x_dtype, YMode mode,
                               const DevInfo& dev, cudaStream_t st) {
    const int engine = g_engine.load(std::memory_order_relaxed);
    const bool streaming = engine == BL_ENGINE_CUDA_CORES || (engine == BL_ENGINE_AUTO && AUTO_ONE_TOKEN_STREAMING);
    if (M == 1 && streaming && gemv1_ok(probs, count, M, dev)) return launch_gemv1(probs, count, x_dtype, mode, dev, st);
    const GemvProblem& q = probs[0];
    if (count == 1 && x_dtype == BL_I8)
        return launch_gemv(static_cast<const int8_t*>(q.x), q.gamma, M, q.K, q.W_p, q.beta, q.N, q.y, mode, dev, st);
    if (count == 1) return launch_gemv_fused(q.x, x_dtype == BL_BF16, M, q.K, q.W_p, q.beta, q.N, q.y, mode, dev, st);
    return launch_gemv_fused_group(probs, count, M, x_dtype, mode, dev, st);
}

cudaError_t ensure_smem_optin(const void* kernel, size_t bytes) {
    static std::mutex mu;
    static std::vector<std::pair<std::pair<const void*, int>, size_t>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (auto& d : done)
        if (d.first.first == kernel && d.first.second == dev && d.second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    for (auto& d : done)
        if (d.first.first == kernel && d.first.second == dev) {
            d.second = bytes;
            return cudaSuccess;
        }
    done.push_back({{kernel, dev}, bytes});
    return cudaSuccess;
}

}  // namespace bl

using namespace bl;

extern "C" {

const char* bitlinear_status_string(bl_status s) {
    switch (s) {
        case BL_OK: return "ok";
        case BL_ERR_NULL: return "null pointer";
        case BL_ERR_SHAPE: return "invalid shape";
        case BL_ERR_ALIGN: return "pointer not 16-byte aligned";
        case BL_ERR_DTYPE: return "invalid dtype or combine mode";
        case BL_ERR_WORKSPACE: return "workspace missing or too small";
        case BL_ERR_DEVICE: return "no compute capability 10.x CUDA device";
        case BL_ERR_CUDA: return "CUDA launch or runtime error";
        case BL_ERR_TIMEOUT: return "bounded device wait expired";
        case BL_ERR_ALIAS: return "output overlaps an input";
    }
    return "unknown status";
}

size_t bitlinear_quantize_weights_workspace(int64_t N, int64_t K) {
    (void)N;
    (void)K;
    return quantize_weights_ws_bytes();
}

bl_status bitlinear_quantize_weights(const float* W, int64_t N, int64_t K, float eps, int8_t* W_t, float* beta,
                                     void* ws, size_t ws_bytes, void* stream) {
    if (!W || !W_t || !beta) return BL_ERR_NULL;
    bl_status s = check_nk(N, K, 16);
    if (s) return s;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return BL_ERR_SHAPE;
    if (!ws || ws_bytes < quantize_weights_ws_bytes()) return BL_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(W_t) || !aligned16(beta) || !aligned16(ws)) return BL_ERR_ALIGN;
    const size_t n = (size_t)N * K;
    if (overlap(W_t, n, W, n * 4) || overlap(beta, 4, W, n * 4) || overlap(W_t, n, beta, 4) ||
        overlap(ws, ws_bytes, W, n * 4) || overlap(ws, ws_bytes, W_t, n) || overlap(ws, ws_bytes, beta, 4))
        return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(launch_quantize_weights(W, (long long)n, eps, W_t, beta, ws, dev.num_sms, as_stream(stream)));
}

bl_status bitlinear_pack(const int8_t* W_t, int64_t N, int64_t K, uint32_t* W_p, void* stream) {
    if (!W_t || !W_p) return BL_ERR_NULL;
    bl_status s = check_nk(N, K, 16);
    if (s) return s;
    if (!aligned16(W_t) || !aligned16(W_p)) return BL_ERR_ALIGN;
    const size_t n = (size_t)N * K;
    if (overlap(W_p, n / 4, W_t, n)) return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(launch_pack(W_t, (long long)(n / 16), W_p, dev.num_sms, as_stream(stream)));
}

size_t bitlinear_binarize_weights_workspace(int64_t N, int64_t K) {
    (void)N;
    (void)K;
    return binarize_weights_ws_bytes();
}

bl_status bitlinear_binarize_weights(const float* W, int64_t N, int64_t K, int8_t* W_b, float* alpha, float* beta,
                                     void* ws, size_t ws_bytes, void* stream) {
    if (!W || !W_b || !alpha || !beta) return BL_ERR_NULL;
    bl_status s = check_nk(N, K, 32);
    if (s) return s;
    if (!ws || ws_bytes < binarize_weights_ws_bytes()) return BL_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(W_b) || !aligned16(alpha) || !aligned16(beta) || !aligned16(ws))
        return BL_ERR_ALIGN;
    const size_t n = (size_t)N * K;
    const void* outs[4] = {W_b, alpha, beta, ws};
    const size_t sizes[4] = {n, 4, 4, ws_bytes};
    for (int i = 0; i < 4; ++i) {
        if (overlap(outs[i], sizes[i], W, n * 4)) return BL_ERR_ALIAS;
        for (int j = i + 1; j < 4; ++j)
            if (overlap(outs[i], sizes[i], outs[j], sizes[j])) return BL_ERR_ALIAS;
    }
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(
        launch_binarize_weights(W, (long long)n, W_b, alpha, beta, ws, dev.num_sms, as_stream(stream)));
}

bl_status bitlinear_pack_bits(const int8_t* W_b, int64_t N, int64_t K, uint32_t* W_p, void* stream) {
    if (!W_b || !W_p) return BL_ERR_NULL;
    bl_status s = check_nk(N, K, 32);
    if (s) return s;
    if (!aligned16(W_b) || !aligned16(W_p)) return BL_ERR_ALIGN;
    const size_t n = (size_t)N * K;
    if (overlap(W_p, n / 8, W_b, n)) return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(launch_pack_bits(W_b, (long long)(n / 32), W_p, dev.num_sms, as_stream(stream)));
}

bl_status bitlinear_quant_act(const void* x, int x_dtype, int64_t M, int64_t K, int8_t* x_q, float* gamma,
                              void* stream) {
    if (!x || !x_q || !gamma) return BL_ERR_NULL;
    if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_DTYPE;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(1, K, 16);
    if (s) return s;
    if (!aligned16(x) || !aligned16(x_q) || !aligned16(gamma)) return BL_ERR_ALIGN;
    const size_t xb = (size_t)M * K * (x_dtype == BL_BF16 ? 2 : 4);
    if (overlap(x_q, (size_t)M * K, x, xb) || overlap(gamma, (size_t)M * 4, x, xb) ||
        overlap(gamma, (size_t)M * 4, x_q, (size_t)M * K))
        return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(launch_quant_act(x, x_dtype == BL_BF16, M, K, x_q, gamma, as_stream(stream)));
}

size_t bitlinear_forward_workspace(int64_t M, int64_t N, int64_t K) {
    if (M <= AUTO_CUDA_MAX_M) return 0;  // larger M may run the GEMM, which needs row sums
    return gemm_ws_bytes(M, N, K);
}

bl_status bitlinear_forward(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, const uint32_t* W_p,
                            const float* beta, int64_t N, void* y, int y_dtype, void* ws, size_t ws_bytes,
                            void* stream) {
    if (y_dtype != BL_F32 && y_dtype != BL_BF16) {
        if (!x_q || !gamma || !W_p || !beta || !y) return BL_ERR_NULL;
        return BL_ERR_DTYPE;
    }
    const size_t ye = y_dtype == BL_F32 ? 4 : 2;
    if (!gamma || !beta) return BL_ERR_NULL;
    bl_status s = check_forward(x_q, gamma, M, K, W_p, beta, N, y, ye);
    if (s) return s;
    return run_forward(x_q, gamma, M, K, W_p, beta, N, y, y_dtype == BL_F32 ? Y_F32 : Y_BF16, ws, ws_bytes, stream);
}

static size_t round256(size_t n) { return (n + 255) / 256 * 256; }

size_t bitlinear_forward_fp_workspace(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || K < 1) return 0;
    if (gemv_fused_quant_ok(M, K)) return 0;
    return round256((size_t)M * K) + round256((size_t)M * 4) + bitlinear_forward_workspace(M, N, K);
}

bl_status bitlinear_forward_fp(const void* x, int x_dtype, int64_t M, int64_t K, const uint32_t* W_p,
                               const float* beta, int64_t N, void* y, int y_dtype, void* ws, size_t ws_bytes,
                               void* stream) {
    if (!x || !W_p || !beta || !y) return BL_ERR_NULL;
    if ((x_dtype != BL_F32 && x_dtype != BL_BF16) || (y_dtype != BL_F32 && y_dtype != BL_BF16)) return BL_ERR_DTYPE;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(N, K, 64);
    if (s) return s;
    if (!aligned16(x) || !aligned16(W_p) || !aligned16(beta) || !aligned16(y)) return BL_ERR_ALIGN;
    const size_t ye = y_dtype == BL_F32 ? 4 : 2;
    const size_t ybytes = (size_t)M * N * ye, xb = (size_t)M * K * (x_dtype == BL_BF16 ? 2 : 4);
    if (overlap(y, ybytes, x, xb) || overlap(y, ybytes, W_p, (size_t)N * (K / 16) * 4) || overlap(y, ybytes, beta, 4))
        return BL_ERR_ALIAS;
    const size_t need = bitlinear_forward_fp_workspace(M, N, K);
    if (need && (!ws || ws_bytes < need)) return BL_ERR_WORKSPACE;
    if (need && !aligned16(ws)) return BL_ERR_ALIGN;
    if (need && (overlap(ws, need, x, xb) || overlap(ws, need, y, ybytes))) return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    const YMode mode = y_dtype == BL_F32 ? Y_F32 : Y_BF16;
    const GemvProblem prob = {x, nullptr, W_p, beta, y, (int)K, (int)N};
    // The swap-AB kernel quantises in its prologue only for a few tokens; from
    // 5 tokens on the standalone quantiser (one CTA per token) plus the kernel
    // on x_q is faster (M = 16: 13 / 22 us instead of 30 / 40 us).
    if (M <= 4 && pick_path((int)M, &prob, 1, dev) == PATH_TC)  // quantiser fused, workspace unused
        return from_cuda(launch_decode_tc(&prob, 1, (int)M, x_dtype, mode, dev, as_stream(stream)));
    if (!need)
        return from_cuda(launch_decode_cuda(&prob, 1, (int)M, x_dtype, mode, dev, as_stream(stream)));
    int8_t* x_q = reinterpret_cast<int8_t*>(ws);
    float* gamma = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + round256((size_t)M * K));
    char* fws = reinterpret_cast<char*>(gamma) + round256((size_t)M * 4);
    // on the tensor-core paths the quantiser also writes the row sums of x_q
    // (at the start of the forward's workspace): the GEMM then needs no
    // row-sum launch and the swap-AB kernel no read-back of x_hat
    const bool rows = pick_path((int)M, &prob, 1, dev) != PATH_CUDA;
    cudaError_t e = launch_quant_act(x, x_dtype == BL_BF16, M, K, x_q, gamma, as_stream(stream),
                                     rows ? reinterpret_cast<int*>(fws) : nullptr);
    if (e != cudaSuccess) return BL_ERR_CUDA;
    return run_forward(x_q, gamma, M, K, W_p, beta, N, y, mode, fws, ws_bytes - (fws - reinterpret_cast<char*>(ws)),
                       stream, rows);
}

bl_status bitlinear_forward_fp_batch(const bl_problem* problems, int count, int64_t M, int x_dtype, int y_dtype,
                                     void* stream) {
    if (!problems) return BL_ERR_NULL;
    if (count < 1 || count > BL_BATCH_MAX || count > gemv_group_max()) return BL_ERR_SHAPE;
    if ((x_dtype != BL_F32 && x_dtype != BL_BF16 && x_dtype != BL_I8) || (y_dtype != BL_F32 && y_dtype != BL_BF16))
        return BL_ERR_DTYPE;
    if (M < 1 || !gemv_fused_quant_ok(M, 64)) return BL_ERR_SHAPE;
    const size_t xe = x_dtype == BL_BF16 ? 2 : x_dtype == BL_I8 ? 1 : 4, ye = y_dtype == BL_F32 ? 4 : 2;
    GemvProblem probs[BL_BATCH_MAX];
    for (int i = 0; i < count; ++i) {
        const bl_problem& q = problems[i];
        if (!q.x || !q.W_p || !q.beta || !q.y || (x_dtype == BL_I8 && !q.gamma)) return BL_ERR_NULL;
        bl_status s = check_nk(q.N, q.K, 64);
        if (s) return s;
        if (!gemv_fused_quant_ok(M, q.K)) return BL_ERR_SHAPE;
        if (!aligned16(q.x) || !aligned16(q.W_p) || !aligned16(q.beta) || !aligned16(q.y) ||
            (x_dtype == BL_I8 && !aligned16(q.gamma)))
            return BL_ERR_ALIGN;
        probs[i] = {q.x, x_dtype == BL_I8 ? q.gamma : nullptr, q.W_p, q.beta, q.y, (int)q.K, (int)q.N};
    }
    for (int i = 0; i < count; ++i) {  // no output overlaps any input or another output
        const bl_problem& a = problems[i];
        const size_t yb = (size_t)M * a.N * ye;
        for (int j = 0; j < count; ++j) {
            const bl_problem& b = problems[j];
            if (overlap(a.y, yb, b.x, (size_t)M * b.K * xe) || overlap(a.y, yb, b.W_p, (size_t)b.N * (b.K / 16) * 4) ||
                (x_dtype == BL_I8 && overlap(a.y, yb, b.gamma, (size_t)M * 4)) ||
                overlap(a.y, yb, b.beta, 4) || (i != j && overlap(a.y, yb, b.y, (size_t)M * b.N * ye)))
                return BL_ERR_ALIAS;
        }
    }
    DevInfo dev;
    bl_status s = current_device(dev);
    if (s) return s;
    const YMode mode = y_dtype == BL_F32 ? Y_F32 : Y_BF16;
    if (pick_path((int)M, probs, count, dev) == PATH_TC)
        return from_cuda(launch_decode_tc(probs, count, (int)M, x_dtype, mode, dev, as_stream(stream)));
    return from_cuda(launch_decode_cuda(probs, count, (int)M, x_dtype, mode, dev, as_stream(stream)));
}

size_t bitlinear_forward_binary_workspace(int64_t M, int64_t N, int64_t K) { return forward_bits_ws(M, N, K); }

bl_status bitlinear_forward_binary(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, const uint32_t* W_p,
                                   const float* beta, int64_t N, void* y, int y_dtype, void* ws, size_t ws_bytes,
                                   void* stream) {
    if (!gamma || !beta) return BL_ERR_NULL;
    if (y_dtype != BL_F32 && y_dtype != BL_BF16) {
        if (!x_q || !W_p || !y) return BL_ERR_NULL;
        return BL_ERR_DTYPE;
    }
    bl_status s = check_forward(x_q, gamma, M, K, W_p, beta, N, y, y_dtype == BL_F32 ? 4 : 2, 1);
    if (s) return s;
    return run_forward_bits(x_q, gamma, M, K, W_p, beta, N, y, y_dtype == BL_F32 ? Y_F32 : Y_BF16, ws, ws_bytes,
                            stream);
}

bl_status bitlinear_forward_binary_acc(const int8_t* x_q, int64_t M, int64_t K, const uint32_t* W_p, int64_t N,
                                       int32_t* acc, void* ws, size_t ws_bytes, void* stream) {
    bl_status s = check_forward(x_q, nullptr, M, K, W_p, nullptr, N, acc, 4, 1);
    if (s) return s;
    return run_forward_bits(x_q, nullptr, M, K, W_p, nullptr, N, acc, Y_ACC, ws, ws_bytes, stream);
}

size_t bitlinear_forward_binary_fp_workspace(int64_t M, int64_t N, int64_t K) {
    if (M < 1 || K < 1 || bits_on_gemv(M, K)) return 0;
    return round256((size_t)M * K) + round256((size_t)M * 4) + forward_bits_ws(M, N, K);
}

bl_status bitlinear_forward_binary_fp(const void* x, int x_dtype, int64_t M, int64_t K, const uint32_t* W_p,
                                      const float* beta, int64_t N, void* y, int y_dtype, void* ws, size_t ws_bytes,
                                      void* stream) {
    if (!x || !W_p || !beta || !y) return BL_ERR_NULL;
    if ((x_dtype != BL_F32 && x_dtype != BL_BF16) || (y_dtype != BL_F32 && y_dtype != BL_BF16)) return BL_ERR_DTYPE;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(N, K, 128);
    if (s) return s;
    if (!aligned16(x) || !aligned16(W_p) || !aligned16(beta) || !aligned16(y)) return BL_ERR_ALIGN;
    const size_t ye = y_dtype == BL_F32 ? 4 : 2;
    const size_t ybytes = (size_t)M * N * ye, xb = (size_t)M * K * (x_dtype == BL_BF16 ? 2 : 4);
    if (overlap(y, ybytes, x, xb) || overlap(y, ybytes, W_p, (size_t)N * K / 8) || overlap(y, ybytes, beta, 4))
        return BL_ERR_ALIAS;
    const size_t need = bitlinear_forward_binary_fp_workspace(M, N, K);
    if (need && (!ws || ws_bytes < need)) return BL_ERR_WORKSPACE;
    if (need && !aligned16(ws)) return BL_ERR_ALIGN;
    if (need && (overlap(ws, need, x, xb) || overlap(ws, need, y, ybytes))) return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    const YMode mode = y_dtype == BL_F32 ? Y_F32 : Y_BF16;
    if (!need)  // quantiser fused into the GEMV prologue
        return from_cuda(launch_gemv_bits(x, x_dtype, nullptr, (int)M, (int)K, W_p, beta, (int)N, y, mode, dev,
                                          as_stream(stream)));
    int8_t* x_q = reinterpret_cast<int8_t*>(ws);
    float* gamma = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + round256((size_t)M * K));
    char* fws = reinterpret_cast<char*>(gamma) + round256((size_t)M * 4);
    cudaError_t e = launch_quant_act(x, x_dtype == BL_BF16, M, K, x_q, gamma, as_stream(stream));
    if (e != cudaSuccess) return BL_ERR_CUDA;
    return run_forward_bits(x_q, gamma, M, K, W_p, beta, N, y, mode, fws,
                            ws_bytes - (size_t)(fws - reinterpret_cast<char*>(ws)), stream);
}

bl_status bitlinear_forward_acc(const int8_t* x_q, int64_t M, int64_t K, const uint32_t* W_p, int64_t N,
                                int32_t* acc, void* ws, size_t ws_bytes, void* stream) {
    bl_status s = check_forward(x_q, nullptr, M, K, W_p, nullptr, N, acc, 4);
    if (s) return s;
    return run_forward(x_q, nullptr, M, K, W_p, nullptr, N, acc, Y_ACC, ws, ws_bytes, stream);
}

bl_status bitlinear_quant_act_rms(const float* a, const float* b, int combine, int64_t M, int64_t K, float* h,
                                  int8_t* x_q, float* gamma, void* stream) {
    if (combine != BL_COMBINE_NONE && combine != BL_COMBINE_ADD && combine != BL_COMBINE_SILU_MUL)
        return BL_ERR_DTYPE;
    if (!a || (combine != BL_COMBINE_NONE && !b)) return BL_ERR_NULL;
    if ((x_q == nullptr) != (gamma == nullptr)) return BL_ERR_NULL;
    if (!x_q && !h) return BL_ERR_NULL;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(1, K, 16);
    if (s) return s;
    if (!aligned16(a) || (b && !aligned16(b)) || (h && !aligned16(h)) || (x_q && !aligned16(x_q)) ||
        (gamma && !aligned16(gamma)))
        return BL_ERR_ALIGN;
    const size_t fb = (size_t)M * K * 4;
    const void* ins[2] = {a, combine != BL_COMBINE_NONE ? b : nullptr};
    for (const void* in : ins) {
        if (!in) continue;
        if (overlap(h, h ? fb : 0, in, fb) || overlap(x_q, x_q ? (size_t)M * K : 0, in, fb) ||
            overlap(gamma, gamma ? (size_t)M * 4 : 0, in, fb))
            return BL_ERR_ALIAS;
    }
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(launch_quant_act_rms(a, combine != BL_COMBINE_NONE ? b : nullptr, combine, M, K, h, x_q, gamma,
                                          as_stream(stream)));
}

size_t bitlinear_glu_workspace(int64_t M, int64_t D, int64_t F) {
    if (M < 1 || D < 1 || F < 1) return 0;
    const size_t fw = std::max(bitlinear_forward_workspace(M, F, D), bitlinear_forward_workspace(M, D, F));
    return round256((size_t)M * D) + round256((size_t)M * 4) + 2 * round256((size_t)M * F * 4) +
           round256((size_t)M * F) + round256((size_t)M * 4) + round256(fw);
}

bl_status bitlinear_glu_forward(const float* x, int64_t M, int64_t D, int64_t F, const uint32_t* W_gate,
                                const float* beta_gate, const uint32_t* W_up, const float* beta_up,
                                const uint32_t* W_down, const float* beta_down, float* y, float* u, void* ws,
                                size_t ws_bytes, void* stream) {
    if (!x || !W_gate || !beta_gate || !W_up || !beta_up || !W_down || !beta_down || !y) return BL_ERR_NULL;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(F, D, 64);
    if (s) return s;
    s = check_nk(D, F, 64);
    if (s) return s;
    const size_t need = bitlinear_glu_workspace(M, D, F);
    if (!ws || ws_bytes < need) return BL_ERR_WORKSPACE;
    const void* ptrs[10] = {x, W_gate, beta_gate, W_up, beta_up, W_down, beta_down, y, u, ws};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return BL_ERR_ALIGN;
    const size_t wgu = (size_t)F * (D / 16) * 4, wd = (size_t)D * (F / 16) * 4;
    const void* ins[7] = {x, W_gate, beta_gate, W_up, beta_up, W_down, beta_down};
    const size_t in_bytes[7] = {(size_t)M * D * 4, wgu, 4, wgu, 4, wd, 4};
    const void* outs[3] = {y, u, ws};
    const size_t out_bytes[3] = {(size_t)M * D * 4, u ? (size_t)M * F * 4 : 0, ws_bytes};
    for (int i = 0; i < 3; ++i) {
        for (int j = 0; j < 7; ++j)
            if (overlap(outs[i], out_bytes[i], ins[j], in_bytes[j])) return BL_ERR_ALIAS;
        for (int j = i + 1; j < 3; ++j)
            if (overlap(outs[i], out_bytes[i], outs[j], out_bytes[j])) return BL_ERR_ALIAS;
    }
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    cudaStream_t st = as_stream(stream);
    char* p = reinterpret_cast<char*>(ws);
    int8_t* xq = reinterpret_cast<int8_t*>(p);
    p += round256((size_t)M * D);
    float* gx = reinterpret_cast<float*>(p);
    p += round256((size_t)M * 4);
    float* gate = reinterpret_cast<float*>(p);
    p += round256((size_t)M * F * 4);
    float* up = reinterpret_cast<float*>(p);
    p += round256((size_t)M * F * 4);
    int8_t* uq = reinterpret_cast<int8_t*>(p);
    p += round256((size_t)M * F);
    float* gu = reinterpret_cast<float*>(p);
    p += round256((size_t)M * 4);
    const size_t fws_bytes = ws_bytes - (size_t)(p - reinterpret_cast<char*>(ws));
    // x -> RMS-normalised codes shared by gate and up
    if (launch_quant_act_rms(x, nullptr, C_NONE, M, D, nullptr, xq, gx, st) != cudaSuccess) return BL_ERR_CUDA;
    // gate and up: one launch over both for a few tokens, else one forward each
    const GemvProblem probs[2] = {{xq, gx, W_gate, beta_gate, gate, (int)D, (int)F},
                                  {xq, gx, W_up, beta_up, up, (int)D, (int)F}};
    if (M <= AUTO_CUDA_MAX_M && gemv_fused_quant_ok(M, D)) {
        cudaError_t e = pick_path((int)M, probs, 2, dev) == PATH_TC
                            ? launch_decode_tc(probs, 2, (int)M, BL_I8, Y_F32, dev, st)
                            : launch_decode_cuda(probs, 2, (int)M, BL_I8, Y_F32, dev, st);
        if (e != cudaSuccess) return BL_ERR_CUDA;
    } else {
        s = run_forward(xq, gx, M, D, W_gate, beta_gate, F, gate, Y_F32, p, fws_bytes, stream);
        if (s) return s;
        s = run_forward(xq, gx, M, D, W_up, beta_up, F, up, Y_F32, p, fws_bytes, stream);
        if (s) return s;
    }
    // u = SiLU(gate) * up, RMS-normalised codes of u
    if (launch_quant_act_rms(gate, up, C_SILU_MUL, M, F, u, uq, gu, st) != cudaSuccess) return BL_ERR_CUDA;
    return run_forward(uq, gu, M, F, W_down, beta_down, D, y, Y_F32, p, fws_bytes, stream);
}

size_t bitlinear_quantize_weights_grouped_workspace(int64_t N, int64_t K, int64_t G) {
    if (N < 1 || !groups_ok(K, G)) return 0;
    return regroup_ws_bytes(N, K) + quantize_weights_ws_bytes();
}

bl_status bitlinear_quantize_weights_grouped(const float* W, int64_t N, int64_t K, int64_t G, float eps,
                                             int8_t* W_t, float* beta, void* ws, size_t ws_bytes, void* stream) {
    if (!W || !W_t || !beta) return BL_ERR_NULL;
    bl_status s = check_nk(N, K, 64);
    if (s) return s;
    if (!groups_ok(K, G)) return BL_ERR_SHAPE;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return BL_ERR_SHAPE;
    const size_t need = bitlinear_quantize_weights_grouped_workspace(N, K, G);
    if (!ws || ws_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(W) || !aligned16(W_t) || !aligned16(beta) || !aligned16(ws)) return BL_ERR_ALIGN;
    const size_t n = (size_t)N * K;
    if (overlap(W_t, n, W, n * 4) || overlap(beta, (size_t)G * 4, W, n * 4) || overlap(W_t, n, beta, (size_t)G * 4) ||
        overlap(ws, ws_bytes, W, n * 4) || overlap(ws, ws_bytes, W_t, n) || overlap(ws, ws_bytes, beta, (size_t)G * 4))
        return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    cudaStream_t st = as_stream(stream);
    float* Wg = reinterpret_cast<float*>(ws);  // [G][N][K/G]
    void* qws = reinterpret_cast<char*>(ws) + regroup_ws_bytes(N, K);
    if (launch_regroup(W, N, K, (int)G, Wg, dev.num_sms, st) != cudaSuccess) return BL_ERR_CUDA;
    const size_t ng = n / (size_t)G;
    for (int64_t g = 0; g < G; ++g)
        if (launch_quantize_weights(Wg + g * ng, (long long)ng, eps, W_t + g * ng, beta + g, qws, dev.num_sms, st) !=
            cudaSuccess)
            return BL_ERR_CUDA;
    return BL_OK;
}

bl_status bitlinear_quant_act_grouped(const void* x, int x_dtype, int64_t M, int64_t K, int64_t G, int8_t* x_q,
                                      float* gamma, void* stream) {
    if (!x || !x_q || !gamma) return BL_ERR_NULL;
    if (x_dtype != BL_F32 && x_dtype != BL_BF16) return BL_ERR_DTYPE;
    if (M < 1 || M > (int64_t)INT32_MAX / BL_MAX_GROUPS) return BL_ERR_SHAPE;
    bl_status s = check_nk(1, K, 64);
    if (s) return s;
    if (!groups_ok(K, G)) return BL_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(x_q) || !aligned16(gamma)) return BL_ERR_ALIGN;
    const size_t xb = (size_t)M * K * (x_dtype == BL_BF16 ? 2 : 4), gb = (size_t)M * G * 4;
    if (overlap(x_q, (size_t)M * K, x, xb) || overlap(gamma, gb, x, xb) || overlap(gamma, gb, x_q, (size_t)M * K))
        return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return from_cuda(launch_quant_act_grouped(x, x_dtype == BL_BF16, M, K, (int)G, x_q, gamma, as_stream(stream)));
}

size_t bitlinear_forward_grouped_workspace(int64_t M, int64_t N, int64_t K, int64_t G) {
    return grouped_ws(M, N, K, G);
}

// shared checks of the grouped forward calls (x_q group-major, W_p group-major)
static bl_status check_grouped(const int8_t* x_q, int64_t M, int64_t K, int64_t G, const uint32_t* W_p, int64_t N,
                               const void* out, size_t out_bytes, void* ws, size_t ws_bytes) {
    if (!x_q || !W_p || !out) return BL_ERR_NULL;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(N, K, 64);
    if (s) return s;
    if (!groups_ok(K, G)) return BL_ERR_SHAPE;
    const size_t need = grouped_ws(M, N, K, G);
    if (!ws || ws_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(x_q) || !aligned16(W_p) || !aligned16(out) || !aligned16(ws)) return BL_ERR_ALIGN;
    if (overlap(out, out_bytes, x_q, (size_t)M * K) || overlap(out, out_bytes, W_p, (size_t)N * K / 4) ||
        overlap(ws, ws_bytes, x_q, (size_t)M * K) || overlap(ws, ws_bytes, W_p, (size_t)N * K / 4) ||
        overlap(ws, ws_bytes, out, out_bytes))
        return BL_ERR_ALIAS;
    return BL_OK;
}

bl_status bitlinear_forward_grouped(const int8_t* x_q, const float* gamma, int64_t M, int64_t K, int64_t G,
                                    const uint32_t* W_p, const float* beta, int64_t N, void* y, int y_dtype, void* ws,
                                    size_t ws_bytes, void* stream) {
    if (!gamma || !beta) return BL_ERR_NULL;
    if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_DTYPE;
    const size_t yb = (size_t)M * N * (y_dtype == BL_F32 ? 4 : 2);
    bl_status s = check_grouped(x_q, M, K, G, W_p, N, y, yb, ws, ws_bytes);
    if (s) return s;
    if (!aligned16(gamma) || !aligned16(beta)) return BL_ERR_ALIGN;
    if (overlap(y, yb, gamma, (size_t)M * G * 4) || overlap(y, yb, beta, (size_t)G * 4) ||
        overlap(ws, ws_bytes, gamma, (size_t)M * G * 4) || overlap(ws, ws_bytes, beta, (size_t)G * 4))
        return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    const long long stride = group_acc_stride(M, N);
    int* acc = reinterpret_cast<int*>(ws);
    char* fws = reinterpret_cast<char*>(ws) + round256z((size_t)stride * G * 4);
    s = run_grouped_acc(x_q, M, K, G, W_p, N, acc, stride, fws, ws_bytes - (size_t)(fws - reinterpret_cast<char*>(ws)),
                        dev, stream);
    if (s) return s;
    return from_cuda(launch_grouped_rescale(acc, stride, gamma, beta, (int)M, (int)N, (int)G, y,
                                            y_dtype == BL_F32 ? Y_F32 : Y_BF16, dev.num_sms, as_stream(stream)));
}

bl_status bitlinear_forward_grouped_acc(const int8_t* x_q, int64_t M, int64_t K, int64_t G, const uint32_t* W_p,
                                        int64_t N, int32_t* acc, void* ws, size_t ws_bytes, void* stream) {
    if (M < 1 || N < 1 || !groups_ok(K, G)) return BL_ERR_SHAPE;
    const long long stride = group_acc_stride(M, N);
    bl_status s = check_grouped(x_q, M, K, G, W_p, N, acc, (size_t)stride * G * 4, ws, ws_bytes);
    if (s) return s;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    return run_grouped_acc(x_q, M, K, G, W_p, N, acc, stride, ws, ws_bytes, dev, stream);
}

size_t bitlinear_forward_grouped_fp_workspace(int64_t M, int64_t N, int64_t K, int64_t G) {
    const size_t f = grouped_ws(M, N, K, G);
    if (!f) return 0;
    return round256((size_t)M * K) + round256((size_t)M * G * 4) + f;
}

bl_status bitlinear_forward_grouped_fp(const void* x, int x_dtype, int64_t M, int64_t K, int64_t G,
                                       const uint32_t* W_p, const float* beta, int64_t N, void* y, int y_dtype,
                                       void* ws, size_t ws_bytes, void* stream) {
    if (!x || !W_p || !beta || !y) return BL_ERR_NULL;
    if ((x_dtype != BL_F32 && x_dtype != BL_BF16) || (y_dtype != BL_F32 && y_dtype != BL_BF16)) return BL_ERR_DTYPE;
    if (M < 1 || M > (int64_t)INT32_MAX / BL_MAX_GROUPS) return BL_ERR_SHAPE;
    bl_status s = check_nk(N, K, 64);
    if (s) return s;
    if (!groups_ok(K, G)) return BL_ERR_SHAPE;
    const size_t need = bitlinear_forward_grouped_fp_workspace(M, N, K, G);
    if (!ws || ws_bytes < need) return BL_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(W_p) || !aligned16(beta) || !aligned16(y) || !aligned16(ws)) return BL_ERR_ALIGN;
    const size_t xb = (size_t)M * K * (x_dtype == BL_BF16 ? 2 : 4), yb = (size_t)M * N * (y_dtype == BL_F32 ? 4 : 2);
    if (overlap(y, yb, x, xb) || overlap(y, yb, W_p, (size_t)N * K / 4) || overlap(y, yb, beta, (size_t)G * 4) ||
        overlap(ws, ws_bytes, x, xb) || overlap(ws, ws_bytes, y, yb))
        return BL_ERR_ALIAS;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    const int64_t Kg = K / G;
    if (M == 1 && gemv_fused_quant_ok(1, Kg)) {
        // One token: group g of x is the contiguous slice x[g*Kg, (g+1)*Kg), so
        // every group is one problem of a fused quantiser + GEMV launch that
        // writes its rescaled binary32 term; a second pass adds them in order.
        const size_t xe = x_dtype == BL_BF16 ? 2 : 4;
        const long long stride = group_acc_stride(M, N);
        float* t = reinterpret_cast<float*>(ws);
        GemvProblem probs[BL_MAX_GROUPS];
        for (int64_t g = 0; g < G; ++g)
            probs[g] = {reinterpret_cast<const char*>(x) + g * Kg * xe, nullptr, W_p + g * N * (Kg / 16), beta + g,
                        t + g * stride, (int)Kg, (int)N};
        const cudaError_t e = pick_path(1, probs, (int)G, dev) == PATH_TC
                                  ? launch_decode_tc(probs, (int)G, 1, x_dtype, Y_F32, dev, as_stream(stream))
                                  : launch_decode_cuda(probs, (int)G, 1, x_dtype, Y_F32, dev, as_stream(stream));
        if (e != cudaSuccess) return BL_ERR_CUDA;
        return from_cuda(launch_grouped_sum(t, stride, N, (int)G, y, y_dtype == BL_F32 ? Y_F32 : Y_BF16, dev.num_sms,
                                            as_stream(stream)));
    }
    int8_t* x_q = reinterpret_cast<int8_t*>(ws);
    float* gamma = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + round256((size_t)M * K));
    char* fws = reinterpret_cast<char*>(gamma) + round256((size_t)M * G * 4);
    if (launch_quant_act_grouped(x, x_dtype == BL_BF16, M, K, (int)G, x_q, gamma, as_stream(stream)) != cudaSuccess)
        return BL_ERR_CUDA;
    return bitlinear_forward_grouped(x_q, gamma, M, K, G, W_p, beta, N, y, y_dtype, fws,
                                     ws_bytes - (size_t)(fws - reinterpret_cast<char*>(ws)), stream);
}

bl_status bitlinear_device_status(void* stream) {
    DevInfo dev;
    bl_status s = current_device(dev);
    if (s) return s;
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return BL_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int)) != cudaSuccess) return BL_ERR_CUDA;
    if (v) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int)) != cudaSuccess) return BL_ERR_CUDA;
        return BL_ERR_TIMEOUT;
    }
    return BL_OK;
}

bl_status bitlinear_set_decode_engine(int engine) {
    if (engine != BL_ENGINE_AUTO && engine != BL_ENGINE_CUDA_CORES && engine != BL_ENGINE_TENSOR_CORES &&
        engine != BL_ENGINE_CUDA_CORES_GENERAL)
        return BL_ERR_SHAPE;
    g_engine.store(engine, std::memory_order_relaxed);
    return BL_OK;
}

int bitlinear_get_decode_engine(void) { return g_engine.load(std::memory_order_relaxed); }

bl_status bitlinear_forward_path(int64_t M, int64_t N, int64_t K, int* path) {
    if (!path) return BL_ERR_NULL;
    if (M < 1 || M > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    bl_status s = check_nk(N, K, 64);
    if (s) return s;
    DevInfo dev;
    s = current_device(dev);
    if (s) return s;
    const GemvProblem prob = {nullptr, nullptr, nullptr, nullptr, nullptr, (int)K, (int)N};
    const DecodePath p = pick_path((int)M, &prob, 1, dev);
    *path = p == PATH_CUDA ? BL_PATH_CUDA_CORES : p == PATH_TC ? BL_PATH_SWAP_AB : BL_PATH_GEMM;
    return BL_OK;
}

bl_status bitlinear_test_expire_next_wait(int enable) {
    g_expire_next_wait.store(enable ? 1 : 0, std::memory_order_relaxed);
    return BL_OK;
}

int bitlinear_num_sms(void) {
    DevInfo dev;
    if (current_device(dev)) return 0;
    return dev.num_sms;
}

}  // extern "C"
