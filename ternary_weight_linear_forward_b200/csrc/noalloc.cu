// noalloc.cu -- bitlinear_forward for callers that cannot allocate device memory.
//
// Some callers of this library have no way to obtain scratch memory: a C
// runtime that owns a fixed arena and hands out no device allocator, code
// recorded into a stream capture where an allocation would break the capture,
// or a host that must not touch the process-wide caching allocator of another
// framework.  The prefill GEMM needs M int32 row sums of x_q as scratch; this
// entry point keeps them in a static device array of this file instead of a
// caller workspace, and otherwise runs the same kernels as bitlinear_forward.
//
// The array is shared by every call on a device and keeps the last call's
// contents.  Each call overwrites the first M entries before reading them, so
// nothing has to start at zero; calls that overlap on the GPU (for example on
// two streams) race on it.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace bl {
namespace {

// Row-sum scratch of the prefill path; its device address comes from
// cudaGetSymbolAddress (in host code the name is only a host-side stand-in).
static __device__ __align__(256) int g_noalloc_rowsum[BL_NOALLOC_MAX_M];

constexpr int NOALLOC_MAX_DEVICES = 64;

struct NoallocDev {
    std::once_flag once;
    bool ok = false;
    void* scratch = nullptr;
    DevInfo info = {0, 0};
};
NoallocDev g_noalloc[NOALLOC_MAX_DEVICES];

// Once per device, with that device current: device checks and the device
// address of the static scratch array.
bl_status noalloc_setup(NoallocDev*& out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= NOALLOC_MAX_DEVICES) {
        cudaGetLastError();
        return BL_ERR_DEVICE;
    }
    NoallocDev& s = g_noalloc[dev];
    std::call_once(s.once, [&]() {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) {
            cudaGetLastError();
            return;
        }
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_rowsum) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return;
        }
        s.scratch = ptr;
        s.info.num_sms = prop.multiProcessorCount;
        s.info.max_smem_optin = (int)prop.sharedMemPerBlockOptin;
        s.ok = true;
    });
    if (!s.ok) return BL_ERR_DEVICE;
    out = &s;
    return BL_OK;
}

bool aligned16_na(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap_na(const void* a, size_t na, const void* b, size_t nb) {
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}


}  // namespace
}  // namespace bl

using namespace bl;

extern "C" bl_status bitlinear_forward_noalloc(const int8_t* x_q, const float* gamma, int64_t M, int64_t K,
                                               const uint32_t* W_p, const float* beta, int64_t N, void* y,
                                               int y_dtype, void* stream) {
    if (!x_q || !gamma || !W_p || !beta || !y) return BL_ERR_NULL;
    if (y_dtype != BL_F32 && y_dtype != BL_BF16) return BL_ERR_DTYPE;
    if (M < 1 || N < 1 || K < 1 || K % 64 != 0 || K > BL_MAX_K || N > (int64_t)INT32_MAX) return BL_ERR_SHAPE;
    if (M > BL_NOALLOC_MAX_M) return BL_ERR_WORKSPACE;  // more rows than the built-in scratch holds
    if (!aligned16_na(x_q) || !aligned16_na(gamma) || !aligned16_na(W_p) || !aligned16_na(beta) || !aligned16_na(y))
        return BL_ERR_ALIGN;
    const size_t ybytes = (size_t)M * N * (y_dtype == BL_F32 ? 4 : 2);
    if (overlap_na(y, ybytes, x_q, (size_t)M * K) || overlap_na(y, ybytes, W_p, (size_t)N * (K / 16) * 4) ||
        overlap_na(y, ybytes, gamma, (size_t)M * 4) || overlap_na(y, ybytes, beta, 4))
        return BL_ERR_ALIAS;
    NoallocDev* d = nullptr;
    bl_status s = noalloc_setup(d);
    if (s) return s;
    const YMode mode = y_dtype == BL_F32 ? Y_F32 : Y_BF16;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    const GemvProblem prob = {x_q, gamma, W_p, beta, y, (int)K, (int)N};
    const DecodePath path = decode_path((int)M, &prob, 1, d->info);
    if (path == PATH_TC)
        e = launch_decode_tc(&prob, 1, (int)M, BL_I8, mode, d->info, st);
    else if (path == PATH_CUDA)
        e = launch_decode_cuda(&prob, 1, (int)M, BL_I8, mode, d->info, st);
    else
        e = launch_gemm(x_q, gamma, (int)M, (int)K, W_p, beta, (int)N, y, mode, d->scratch, d->info, st, 2,
                        false);  // the static scratch holds row sums only: no split along K
    return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}
